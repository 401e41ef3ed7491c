/*
 * avq_oracle.c -- plain, slow, fp64 CPU oracle for the AVQ-attention forward
 * path ("AVQ-Attention: Adaptive Vector-Quantized Attention").
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or
 * call this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg do. It shares no code with the CUDA kernels.
 *
 * Every input arrives as fp64 holding the exact value of the stored element
 * (bf16 and fp32 widen exactly). Every sum runs in index order, in fp64, and
 * the file is compiled with -ffp-contract=off so that no multiply-add is
 * fused: the result of each function is a fixed function of its inputs.
 *
 * Shapes (row-major, contiguous):
 *   K, V, Q, O : [B, H, N, d]
 *   codebook   : [H, Mtot, d], Mtot = M0*(1+C), tree order: parents 0..M0-1,
 *                child c of parent p at row M0 + p*C + c
 *   assign     : [B, H, N]        leaf id in tree order
 *   counts     : [B, H, Mtot]     int64
 *   vsum       : [B, H, Mtot, d]
 *
 * Readings of points the paper leaves open:
 *   - argmin ties go to the lowest index; a child replaces the parent only
 *     when strictly closer ("reassigned if a child is closer than the
 *     (cached) parent distance", paper §4.2);
 *   - a parent's statistics cover its whole cluster, a child's only the keys
 *     reassigned to it (papernotes summary, design 2);
 *   - codewords with count 0 carry no weight and are left out of the
 *     stabilising maximum;
 *   - importance uses the parent-only denominator of each query (paper §4.3
 *     "Codeword importance"; exact because every parent is on chip);
 *   - selection is the P largest importances, ties to the lower parent index,
 *     listed by descending importance;
 *   - logits are scale * Q_i . C_j (the paper writes exp(Q C^T) with any
 *     scale folded into Q).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OK 0
#define EINVAL_ (-1)
#define ENOMEM_ (-3)

/* Squared Euclidean distance ||a - b||^2, terms summed in index order
 * (paper §3.2: a(K_j) = argmin_a ||C_a - K_j||^2). */
static double sq_dist(const double* a, const double* b, int d) {
    double s = 0.0;
    for (int j = 0; j < d; ++j) {
        double t = a[j] - b[j];
        s += t * t;
    }
    return s;
}

/* Dot product a . b in index order. */
static double dot(const double* a, const double* b, int d) {
    double s = 0.0;
    for (int j = 0; j < d; ++j) s += a[j] * b[j];
    return s;
}

/*
 * Fused full-tree VQ precompute (paper §4.2 "Vector Quantization for
 * (A)VQ-Attention"; papernotes summary, design 2):
 *   1. each key goes to its nearest parent among the M0 roots, and that
 *      distance is kept;
 *   2. the key is compared against only the C children of that parent and
 *      moves to a child if the child is closer than the kept distance;
 *   3. at each level the key's value and a count are added to the codeword it
 *      belongs to: the parent always (its whole cluster), the child only when
 *      the key moved.
 * dist_evals (nullable) receives the number of distance evaluations, which is
 * N*(M0+C) per head (paper Table 1, "VQ assignment" row).
 */
int oracle_precompute(int B, int H, int N, int d, int M0, int C,
                      const double* K, const double* V, const double* codebook,
                      int32_t* assign, int64_t* counts, double* vsum,
                      int64_t* dist_evals, int nthreads) {
    if (B < 0 || H < 0 || N < 0 || d <= 0 || M0 <= 0 || C < 0) return EINVAL_;
    const int Mtot = M0 * (1 + C);
    const int64_t BH = (int64_t)B * H;
    int64_t evals = 0;
    if (nthreads <= 0) nthreads = 1;

    /* steps 1-2: assignment, independent per key */
    const int64_t R = BH * (int64_t)N;
#pragma omp parallel for schedule(static) num_threads(nthreads) reduction(+ : evals)
    for (int64_t r = 0; r < R; ++r) {
        const int64_t bh = r / N;
        const int h = (int)(bh % H);
        const double* k = K + r * d;
        const double* cb = codebook + (int64_t)h * Mtot * d;
        int best_p = 0;
        double best = sq_dist(k, cb, d);
        for (int p = 1; p < M0; ++p) {
            double dd = sq_dist(k, cb + (int64_t)p * d, d);
            if (dd < best) { best = dd; best_p = p; }
        }
        int leaf = best_p;
        double leaf_d = best;               /* cached parent distance */
        for (int c = 0; c < C; ++c) {
            int idx = M0 + best_p * C + c;
            double dd = sq_dist(k, cb + (int64_t)idx * d, d);
            if (dd < leaf_d) { leaf_d = dd; leaf = idx; }
        }
        assign[r] = leaf;
        evals += M0 + C;
    }
    if (dist_evals) *dist_evals = evals;

    /* step 3: aggregation, keys in index order (deterministic) */
#pragma omp parallel for schedule(static) num_threads(nthreads)
    for (int64_t bh = 0; bh < BH; ++bh) {
        int64_t* cnt = counts + bh * Mtot;
        double* vs = vsum + bh * (int64_t)Mtot * d;
        memset(cnt, 0, sizeof(int64_t) * (size_t)Mtot);
        memset(vs, 0, sizeof(double) * (size_t)Mtot * (size_t)d);
        for (int n = 0; n < N; ++n) {
            const int64_t r = bh * N + n;
            const int leaf = assign[r];
            const int parent = leaf < M0 ? leaf : (leaf - M0) / (C > 0 ? C : 1);
            const double* v = V + r * d;
            cnt[parent] += 1;
            for (int j = 0; j < d; ++j) vs[(int64_t)parent * d + j] += v[j];
            if (leaf != parent) {
                cnt[leaf] += 1;
                for (int j = 0; j < d; ++j) vs[(int64_t)leaf * d + j] += v[j];
            }
        }
    }
    return OK;
}

/* Order: larger importance first, ties to the lower parent index. */
static int before(const double* w, int a, int b) {
    if (w[a] > w[b]) return 1;
    if (w[a] < w[b]) return 0;
    return a < b;
}

/*
 * Tiled adaptive attention for one query tile (paper §4.3; papernotes
 * summary, design 3):
 *   1. parent attention: S_ip = scale * Q_i . C_p, A_ip = exp(S_ip - m_i),
 *      Zbar_i = sum_p A_ip n_p;
 *   2. importance w_p(I) = sum_{i in I} A_ip n_p / Zbar_i ("Codeword
 *      importance"); the normalised score w_p / |I| is the fraction of the
 *      tile's attention mass on parent p;
 *   3. the P parents of largest importance are selected ("Child spawning");
 *   4. output: every parent contributes exp(S_ip) [Vbar_p, n_p]; for each
 *      selected parent p and child c the correction
 *      DeltaA_ic = exp(S_ic) - exp(S_ip) is applied to [Vbar_c, n_c]
 *      ("Child attention"; the DeltaA display of the papernotes summary),
 *      all terms under one common shift M_i;  Y_i = Xbar_i / Zbar_i.
 * With parent_logit_from_children != 0 the parent logit inside the
 * correction is the mean of its children's logits (paper §4.3 "Child
 * attention" identity, valid under the parent-child constraint).
 */
static void attention_tile(int d, int M0, int C, int P, int T, int N, double scale,
                           const double* Qbh, const double* cb, const int64_t* cnt,
                           const double* vs, int tile, const int32_t* forced,
                           int parent_logit_from_children,
                           double* O_tile, int32_t* sel_out, double* score_out,
                           int64_t* logit_evals,
                           double* S, double* A, double* Zbar, double* w, int* order,
                           double* Sc) {
    const int i0 = tile * T;
    const int rows = (N - i0) < T ? (N - i0) : T;

    /* 1. parent attention */
    for (int r = 0; r < rows; ++r) {
        const double* q = Qbh + (int64_t)(i0 + r) * d;
        double m = -INFINITY;
        for (int p = 0; p < M0; ++p) {
            S[r * M0 + p] = scale * dot(q, cb + (int64_t)p * d, d);
            if (cnt[p] > 0 && S[r * M0 + p] > m) m = S[r * M0 + p];
        }
        double z = 0.0;
        for (int p = 0; p < M0; ++p) {
            double a = cnt[p] > 0 ? exp(S[r * M0 + p] - m) : 0.0;
            A[r * M0 + p] = a;
            z += a * (double)cnt[p];
        }
        Zbar[r] = z;
        *logit_evals += M0;
    }

    /* 2. importance */
    for (int p = 0; p < M0; ++p) {
        double s = 0.0;
        for (int r = 0; r < rows; ++r) s += A[r * M0 + p] * (double)cnt[p] / Zbar[r];
        w[p] = s;
        score_out[p] = rows > 0 ? s / (double)rows : 0.0;
    }

    /* 3. top-P selection (stable insertion sort by (-w, p)) */
    if (forced) {
        for (int j = 0; j < P; ++j) order[j] = forced[j];
    } else {
        for (int p = 0; p < M0; ++p) {
            int j = p;
            while (j > 0 && before(w, p, order[j - 1])) { order[j] = order[j - 1]; --j; }
            order[j] = p;
        }
    }
    for (int j = 0; j < P; ++j) sel_out[j] = order[j];

    /* 4. output with child correction */
    for (int r = 0; r < rows; ++r) {
        const double* q = Qbh + (int64_t)(i0 + r) * d;
        double M = -INFINITY;
        for (int p = 0; p < M0; ++p)
            if (cnt[p] > 0 && S[r * M0 + p] > M) M = S[r * M0 + p];
        for (int j = 0; j < P; ++j) {
            const int p = order[j];
            for (int c = 0; c < C; ++c) {
                const int idx = M0 + p * C + c;
                double s = scale * dot(q, cb + (int64_t)idx * d, d);
                Sc[j * C + c] = s;
                if (cnt[idx] > 0 && s > M) M = s;
            }
        }
        *logit_evals += (int64_t)P * C;
        double* o = O_tile + (int64_t)r * d;
        for (int k = 0; k < d; ++k) o[k] = 0.0;
        double den = 0.0;
        for (int p = 0; p < M0; ++p) {
            if (cnt[p] <= 0) continue;
            double e = exp(S[r * M0 + p] - M);
            const double* v = vs + (int64_t)p * d;
            for (int k = 0; k < d; ++k) o[k] += e * v[k];
            den += e * (double)cnt[p];
        }
        for (int j = 0; j < P; ++j) {
            const int p = order[j];
            double sp = S[r * M0 + p];
            if (parent_logit_from_children && C > 0) {
                double acc = 0.0;
                for (int c = 0; c < C; ++c) acc += Sc[j * C + c];
                sp = acc / (double)C;
            }
            const double ep = exp(sp - M);
            for (int c = 0; c < C; ++c) {
                const int idx = M0 + p * C + c;
                if (cnt[idx] <= 0) continue;
                const double dA = exp(Sc[j * C + c] - M) - ep;
                const double* v = vs + (int64_t)idx * d;
                for (int k = 0; k < d; ++k) o[k] += dA * v[k];
                den += dA * (double)cnt[idx];
            }
        }
        for (int k = 0; k < d; ++k) o[k] /= den;
    }
    for (int r = rows; r < T; ++r)
        for (int k = 0; k < d; ++k) O_tile[(int64_t)r * d + k] = 0.0;
}

/*
 * Attention over a list of query tiles. A tile id is bh * ntiles + t with
 * ntiles = ceil(N / T); tile_ids == NULL means every tile in order.
 * Outputs are per listed tile:
 *   O        [n, T, d]   rows past N are zero
 *   selected [n, P]      by descending importance, ties to the lower index
 *   score    [n, M0]     w_p / |I| (tile attention-mass fraction)
 * forced (nullable, [n, P]) replaces the selection by a given parent list.
 * logit_evals (nullable) receives the number of query-codeword logits
 * evaluated: (M0 + P*C) per query.
 */
int oracle_attention(int B, int H, int N, int d, int M0, int C,
                     const double* Q, const double* codebook, const int64_t* counts,
                     const double* vsum, int P, int T, double scale,
                     const int32_t* tile_ids, int n_tile_ids, const int32_t* forced,
                     int parent_logit_from_children,
                     double* O, int32_t* selected, double* score, int64_t* logit_evals,
                     int nthreads) {
    if (B < 0 || H < 0 || N < 0 || d <= 0 || M0 <= 0 || C < 0 || T <= 0) return EINVAL_;
    if (P < 0 || P > M0) return EINVAL_;
    const int Mtot = M0 * (1 + C);
    const int ntiles = (N + T - 1) / T;
    const int64_t total = (int64_t)B * H * ntiles;
    const int64_t n = tile_ids ? (int64_t)n_tile_ids : total;
    for (int64_t j = 0; tile_ids && j < n; ++j)
        if (tile_ids[j] < 0 || tile_ids[j] >= total) return EINVAL_;
    if (nthreads <= 0) nthreads = 1;
    int64_t evals = 0;
    int fail = 0;

#pragma omp parallel num_threads(nthreads) reduction(+ : evals)
    {
        double* S = (double*)malloc(sizeof(double) * (size_t)T * (size_t)M0);
        double* A = (double*)malloc(sizeof(double) * (size_t)T * (size_t)M0);
        double* Zbar = (double*)malloc(sizeof(double) * (size_t)T);
        double* w = (double*)malloc(sizeof(double) * (size_t)M0);
        int* order = (int*)malloc(sizeof(int) * (size_t)M0);
        double* Sc = (double*)malloc(sizeof(double) * (size_t)(P * C > 0 ? P * C : 1));
        if (!S || !A || !Zbar || !w || !order || !Sc) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t j = 0; j < n; ++j) {
                const int64_t g = tile_ids ? tile_ids[j] : j;
                const int64_t bh = g / ntiles;
                const int t = (int)(g % ntiles);
                const int h = (int)(bh % H);
                attention_tile(d, M0, C, P, T, N, scale, Q + bh * (int64_t)N * d,
                               codebook + (int64_t)h * Mtot * d, counts + bh * Mtot,
                               vsum + bh * (int64_t)Mtot * d, t,
                               forced ? forced + j * P : NULL, parent_logit_from_children,
                               O + j * (int64_t)T * d, selected + j * P, score + j * M0,
                               &evals, S, A, Zbar, w, order, Sc);
            }
        }
        free(S); free(A); free(Zbar); free(w); free(order); free(Sc);
    }
    if (logit_evals) *logit_evals = evals;
    return fail ? ENOMEM_ : OK;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
