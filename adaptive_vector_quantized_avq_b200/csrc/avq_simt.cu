// avq_simt.cu -- CUDA-core (SIMT) kernels of the AVQ-attention forward path.
//
// These kernels compute in fp32 on the CUDA cores. They are the path for
// fp32 inputs, whose logits and distances must not be rounded to a
// tensor-core input format, and serve any shape the tensor-core kernels do
// not take. Decisions (assignments) are those of exact fp64 arithmetic: an
// fp32 filter with a rigorous error bound, then an fp64 re-decision in the
// rare cases the bound does not separate the candidates.
#include "avq_internal.cuh"

namespace avq {

// ---------------------------------------------------------------------------
// Fused full-tree precompute (paper §4.2; papernotes, Key Designs 2).
// One thread per key; the head's parents live in shared memory as fp32, the
// C children of the chosen parent are read through the L1 cache. Counts are
// privatised per CTA in shared memory and flushed with one atomic per
// non-empty codeword; value sums go to global memory with fp32 atomics.
// ---------------------------------------------------------------------------
template <typename T, int D>
__device__ __forceinline__ float dist_f32(const float (&k)[D], const float* c) {
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < D; ++j) {
        float t = __fsub_rn(k[j], c[j]);
        acc = __fmaf_rn(t, t, acc);
    }
    return acc;
}

template <typename T, int D>
__device__ __forceinline__ float dist_f32_global(const float (&k)[D], const T* c) {
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < D; ++j) {
        float t = __fsub_rn(k[j], ld_f32(c + j));
        acc = __fmaf_rn(t, t, acc);
    }
    return acc;
}

template <typename T, int D>
__global__ void __launch_bounds__(128)
precompute_simt_kernel(const T* __restrict__ K, const T* __restrict__ V,
                       const T* __restrict__ codebook, int32_t* __restrict__ assign,
                       int32_t* __restrict__ counts, float* __restrict__ vsum,
                       int H, int N, int M0, int C, int keys_per_cta) {
    extern __shared__ float4 smem_f4[];
    float* par = reinterpret_cast<float*>(smem_f4);          // [M0][D]
    int* cnt = reinterpret_cast<int*>(par + M0 * D);          // [Mtot]
    const int Mtot = M0 * (1 + C);
    const int bh = blockIdx.y;
    const int h = bh % H;
    const T* cb = codebook + (size_t)h * Mtot * D;
    for (int i = threadIdx.x; i < M0 * D; i += blockDim.x) par[i] = ld_f32(cb + i);
    for (int i = threadIdx.x; i < Mtot; i += blockDim.x) cnt[i] = 0;
    __syncthreads();

    const float eps = dist_eps(D);
    const int n0 = blockIdx.x * keys_per_cta;
    const int n1 = min(N, n0 + keys_per_cta);
    for (int n = n0 + threadIdx.x; n < n1; n += blockDim.x) {
        const size_t row = (size_t)bh * N + n;
        const T* kp = K + row * D;
        float k[D];
#pragma unroll
        for (int j = 0; j < D; ++j) k[j] = ld_f32(kp + j);

        // a1: nearest parent; best and runner-up approximate distances
        float best = INFINITY, second = INFINITY;
        int bp = 0;
        for (int p = 0; p < M0; ++p) {
            float dd = dist_f32<T, D>(k, par + p * D);
            if (dd < best) { second = best; best = dd; bp = p; }
            else if (dd < second) { second = dd; }
        }
        if (M0 > 1 && !separated(best, second, eps)) {
            // re-decide in fp64 among the parents the bound cannot separate
            double ebest = INFINITY;
            int ep = -1;
            for (int p = 0; p < M0; ++p) {
                float dd = dist_f32<T, D>(k, par + p * D);
                if (separated(best, dd, eps)) continue;
                double e = exact_sq_dist(kp, cb + (size_t)p * D, D);
                if (e < ebest) { ebest = e; ep = p; }
            }
            if (ep >= 0) bp = ep;   // ep < 0 only for non-finite inputs
            best = dist_f32<T, D>(k, par + bp * D);
        }

        // a2: children of the chosen parent against the kept parent distance
        int leaf = bp;
        if (C > 0) {
            const T* ch = cb + (size_t)(M0 + bp * C) * D;
            float lo = best;
            int lo_idx = -1;  // -1 = parent
            for (int c = 0; c < C; ++c) {
                float dd = dist_f32_global<T, D>(k, ch + (size_t)c * D);
                if (dd < lo) { lo = dd; lo_idx = c; }
            }
            // is the winner separated from every other candidate?
            bool sure = (lo_idx < 0) || separated(lo, best, eps);
            if (sure) {
                for (int c = 0; c < C && sure; ++c) {
                    if (c == lo_idx) continue;
                    float dd = dist_f32_global<T, D>(k, ch + (size_t)c * D);
                    if (!separated(lo, dd, eps)) sure = false;
                }
            }
            if (sure) {
                leaf = lo_idx < 0 ? bp : M0 + bp * C + lo_idx;
            } else {
                // exact rule among the band: parent first, then children in
                // index order, a candidate wins only when strictly closer
                double eb = exact_sq_dist(kp, cb + (size_t)bp * D, D);
                int win = bp;
                for (int c = 0; c < C; ++c) {
                    float dd = dist_f32_global<T, D>(k, ch + (size_t)c * D);
                    if (separated(lo, dd, eps)) continue;
                    double e = exact_sq_dist(kp, ch + (size_t)c * D, D);
                    if (e < eb) { eb = e; win = M0 + bp * C + c; }
                }
                leaf = win;
            }
        }
        assign[row] = leaf;

        // a3: scatter at each level -- the parent always, the child when moved
        atomicAdd(&cnt[bp], 1);
        const T* vp = V + row * D;
        float* dst_p = vsum + ((size_t)bh * Mtot + bp) * D;
        if (leaf != bp) {
            atomicAdd(&cnt[leaf], 1);
            float* dst_c = vsum + ((size_t)bh * Mtot + leaf) * D;
            for (int j = 0; j < D; ++j) {
                float v = ld_f32(vp + j);
                atomicAdd(dst_p + j, v);
                atomicAdd(dst_c + j, v);
            }
        } else {
            for (int j = 0; j < D; ++j) atomicAdd(dst_p + j, ld_f32(vp + j));
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < Mtot; i += blockDim.x)
        if (cnt[i]) atomicAdd(&counts[(size_t)bh * Mtot + i], cnt[i]);
}

// ---------------------------------------------------------------------------
// Tiled adaptive attention (paper §4.3; papernotes, Key Designs 3).
// One CTA per query tile, one thread per query row. Parent codewords, parent
// value sums and counts live in shared memory (fp32); the tile's parent
// weights are kept in shared memory for the importance reduction. Children
// of the selected parents are read through L1. The output accumulates
// online: one running shift per row, rescaled when a child logit exceeds it.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(128)
attention_simt_kernel(const T* __restrict__ Q, const T* __restrict__ codebook,
                      const int32_t* __restrict__ counts, const float* __restrict__ vsum,
                      T* __restrict__ O, int32_t* __restrict__ selected,
                      int H, int N, int M0, int C, int P, int tile, float scale, int ntiles) {
    extern __shared__ float4 smem_f4[];
    float* par = reinterpret_cast<float*>(smem_f4);   // [M0][D]
    float* vpar = par + M0 * D;                         // [M0][D]
    float* npar = vpar + M0 * D;                        // [M0]
    float* w = npar + M0;                               // [M0]
    float* rz = w + M0;                                 // [128]
    int* sel = reinterpret_cast<int*>(rz + 128);        // [M0]
    float* A = reinterpret_cast<float*>(sel + M0);      // [128][M0+1]
    const int lda = M0 + 1;

    const int Mtot = M0 * (1 + C);
    const int t = blockIdx.x;
    const int bh = blockIdx.y;
    const int h = bh % H;
    const T* cb = codebook + (size_t)h * Mtot * D;
    const int32_t* cnt = counts + (size_t)bh * Mtot;
    const float* vs = vsum + (size_t)bh * Mtot * D;
    for (int i = threadIdx.x; i < M0 * D; i += blockDim.x) {
        par[i] = ld_f32(cb + i);
        vpar[i] = vs[i];
    }
    for (int i = threadIdx.x; i < M0; i += blockDim.x) npar[i] = (float)cnt[i];
    __syncthreads();

    const int i0 = t * tile;
    const int rows = min(tile, N - i0);
    const int r = threadIdx.x;
    const bool valid = r < rows;
    float q[D];
    float m = -INFINITY;
    if (valid) {
        const T* qp = Q + ((size_t)bh * N + i0 + r) * D;
#pragma unroll
        for (int j = 0; j < D; ++j) q[j] = ld_f32(qp + j);
        // a4: parent logits and count-weighted denominator
        for (int p = 0; p < M0; ++p) {
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < D; ++j) s = __fmaf_rn(q[j], par[p * D + j], s);
            s *= scale;
            A[r * lda + p] = s;
            if (npar[p] > 0.f && s > m) m = s;
        }
        float z = 0.f;
        for (int p = 0; p < M0; ++p) {
            float a = npar[p] > 0.f ? expf(A[r * lda + p] - m) : 0.f;
            A[r * lda + p] = a;
            z = __fmaf_rn(a, npar[p], z);
        }
        rz[r] = 1.f / z;
    }
    __syncthreads();

    // a5: importance w_p = n_p * sum_i A_ip / Zbar_i
    for (int p = threadIdx.x; p < M0; p += blockDim.x) {
        float s = 0.f;
        for (int i = 0; i < rows; ++i) s = __fmaf_rn(A[i * lda + p], rz[i], s);
        w[p] = s * npar[p];
    }
    __syncthreads();

    // a6: top-P by rank (descending w, ties to the lower index)
    for (int p = threadIdx.x; p < M0; p += blockDim.x) {
        const float wp = w[p];
        int rank = 0;
        for (int q2 = 0; q2 < M0; ++q2) {
            const float wq = w[q2];
            rank += (wq > wp) || (wq == wp && q2 < p);
        }
        if (rank < P) {
            sel[rank] = p;
            selected[((size_t)bh * ntiles + t) * P + rank] = p;
        }
    }
    __syncthreads();

    if (!valid) return;
    // a4 output part: every non-empty parent with its whole cluster
    float num[D];
#pragma unroll
    for (int j = 0; j < D; ++j) num[j] = 0.f;
    float den = 0.f;
    for (int p = 0; p < M0; ++p) {
        const float a = A[r * lda + p];
        if (a == 0.f) continue;
#pragma unroll
        for (int j = 0; j < D; ++j) num[j] = __fmaf_rn(a, vpar[p * D + j], num[j]);
        den = __fmaf_rn(a, npar[p], den);
    }
    // a7: children of the selected parents, DeltaA = e^{S_ic} - e^{S_ip}
    float Mrow = m;         // current shift of num/den
    float pscale = 1.f;     // e^{m - Mrow}: converts parent weights to the current shift
    for (int jsel = 0; jsel < P; ++jsel) {
        const int p = sel[jsel];
        const float ap = A[r * lda + p];
        for (int c = 0; c < C; ++c) {
            const int idx = M0 + p * C + c;
            const int nc = __ldg(cnt + idx);
            if (nc == 0) continue;
            const T* crow = cb + (size_t)idx * D;
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < D; ++j) s = __fmaf_rn(q[j], ld_f32(crow + j), s);
            s *= scale;
            if (s > Mrow) {
                const float f = expf(Mrow - s);
#pragma unroll
                for (int j = 0; j < D; ++j) num[j] *= f;
                den *= f;
                pscale *= f;
                Mrow = s;
            }
            const float dA = expf(s - Mrow) - ap * pscale;
            const float* vrow = vs + (size_t)idx * D;
#pragma unroll
            for (int j = 0; j < D; ++j) num[j] = __fmaf_rn(dA, __ldg(vrow + j), num[j]);
            den = __fmaf_rn(dA, (float)nc, den);
        }
    }
    // a8: Y = Xbar / Zbar
    const float inv = 1.f / den;
    T* op = O + ((size_t)bh * N + i0 + r) * D;
#pragma unroll
    for (int j = 0; j < D; ++j) st_elem(op + j, num[j] * inv);
}

// ------------------------------------------------------------------ launchers
template <typename T, int D>
static cudaError_t launch_precompute_simt_t(const avq_shape& s, const void* K, const void* V,
                                            const void* cb, int32_t* assign, int32_t* counts,
                                            float* vsum, cudaStream_t st) {
    const int keys_per_cta = 1024;
    const int Mtot = s.M0 * (1 + s.C);
    const size_t smem = sizeof(float) * (size_t)s.M0 * D + sizeof(int) * (size_t)Mtot;
    auto kern = precompute_simt_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((s.N + keys_per_cta - 1) / keys_per_cta, s.B * s.H);
    kern<<<grid, 128, smem, st>>>(static_cast<const T*>(K), static_cast<const T*>(V),
                                  static_cast<const T*>(cb), assign, counts, vsum, s.H, s.N,
                                  s.M0, s.C, keys_per_cta);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_precompute_simt(const avq_shape& s, const void* K, const void* V,
                                   const void* cb, int32_t* assign, int32_t* counts,
                                   float* vsum, cudaStream_t st) {
    if (s.dtype == AVQ_F32) {
        if (s.d == 64) return launch_precompute_simt_t<float, 64>(s, K, V, cb, assign, counts, vsum, st);
        return launch_precompute_simt_t<float, 128>(s, K, V, cb, assign, counts, vsum, st);
    }
    if (s.d == 64)
        return launch_precompute_simt_t<__nv_bfloat16, 64>(s, K, V, cb, assign, counts, vsum, st);
    return launch_precompute_simt_t<__nv_bfloat16, 128>(s, K, V, cb, assign, counts, vsum, st);
}

size_t attention_simt_smem(const avq_shape& s) {
    return sizeof(float) * ((size_t)2 * s.M0 * s.d + 2 * s.M0 + 128) + sizeof(int) * s.M0 +
           sizeof(float) * 128 * (size_t)(s.M0 + 1);
}

template <typename T, int D>
static cudaError_t launch_attention_simt_t(const avq_shape& s, const void* Q, const void* cb,
                                           const int32_t* counts, const float* vsum, int P,
                                           int tile, float scale, void* O, int32_t* selected,
                                           cudaStream_t st) {
    const size_t smem = attention_simt_smem(s);
    auto kern = attention_simt_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int ntiles = (s.N + tile - 1) / tile;
    dim3 grid(ntiles, s.B * s.H);
    kern<<<grid, 128, smem, st>>>(static_cast<const T*>(Q), static_cast<const T*>(cb), counts,
                                  vsum, static_cast<T*>(O), selected, s.H, s.N, s.M0, s.C, P,
                                  tile, scale, ntiles);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_attention_simt(const avq_shape& s, const void* Q, const void* cb,
                                  const int32_t* counts, const float* vsum, int P, int tile,
                                  float scale, void* O, int32_t* selected, cudaStream_t st) {
    if (s.dtype == AVQ_F32) {
        if (s.d == 64)
            return launch_attention_simt_t<float, 64>(s, Q, cb, counts, vsum, P, tile, scale, O, selected, st);
        return launch_attention_simt_t<float, 128>(s, Q, cb, counts, vsum, P, tile, scale, O, selected, st);
    }
    if (s.d == 64)
        return launch_attention_simt_t<__nv_bfloat16, 64>(s, Q, cb, counts, vsum, P, tile, scale, O, selected, st);
    return launch_attention_simt_t<__nv_bfloat16, 128>(s, Q, cb, counts, vsum, P, tile, scale, O, selected, st);
}

}  // namespace avq
