// avq_deep.cu -- AVQ attention over codebook trees deeper than parent ->
// child (the extension the paper proposes in §6 "Discussion and Conclusion":
// every further level adds P*C codes to the attention cost per query and
// multiplies the codebook's resolution by C).
//
// The two-level steps carried down every level:
//   * layout: M0 nodes at level 0, M0*C^l at level l; node j of level l has
//     the children j*C + c of level l + 1; rows stored level after level
//     (depth 2 is the [parents | M0 + p*C + c] layout of avq_precompute);
//   * assignment (paper §4.2): nearest level-0 node, then level by level the
//     nearest child of the current node replaces it only when strictly
//     closer (ties to the lower index at every step); the descent stops at
//     the first level where no child is closer;
//   * statistics: every node on a key's path counts the key and sums its
//     value row (the "parent holds its whole cluster" rule at every level);
//   * attention (paper §4.3), per query tile, one shift per row (the
//     largest level-0 log-count logit): level-0 weights, then per expanded
//     level l the candidates (level 0: every level-0 node; deeper: the
//     children of the nodes expanded at l - 1) get the importance
//     sum_i A_ic n_c / Zbar_i with the Zbar of the approximation so far, the
//     P_l largest are expanded (ties to the lower row id), and every child g
//     of an expanded node f adds (A_g - A_f) [vsum_g, n_g] to Xbar and Zbar.
//
// Both kernels run on CUDA cores. The precompute takes one thread per key
// and decides every comparison on fp32 distances, again on exact fp64 ones
// (summed in index order) wherever the fp32 error bound cannot, so its
// decisions are the exact ones. The attention takes
// one CTA per query tile (one thread per row) with the row's Xbar in
// registers and the per-candidate weights in shared memory.
#include <algorithm>

#include "avq_internal.cuh"

namespace avq {
namespace {

constexpr int kMaxL = 4;       // levels of a tree (level 0 .. 3)
constexpr int kCand = 128;     // candidates per level held on chip
constexpr float kRescale = 64.f;   // largest weight exponent (log2) before a row's shift moves
constexpr int kCh = 4;         // children per node whose distances the precompute keeps in registers

struct DeepTree {
    int M0, C, L, Mtot;
    int off[kMaxL + 1];        // first row of each level; off[L] = Mtot
};

DeepTree make_tree(int M0, int C, int L) {
    DeepTree t{};
    t.M0 = M0;
    t.C = C;
    t.L = L;
    long long acc = 0, width = M0;
    for (int l = 0; l < L; ++l) {
        t.off[l] = (int)acc;
        acc += width;
        width *= C;
    }
    t.off[L] = (int)acc;
    t.Mtot = (int)acc;
    return t;
}

long long deep_rows(int M0, int C, int L) {
    long long acc = 0, width = M0;
    for (int l = 0; l < L; ++l) {
        acc += width;
        width *= C;
    }
    return acc;
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// element e (0 .. 4 / sizeof(T) - 1) of a 32-bit word of T values, as fp64
// (exact: bf16 and fp32 values widen without rounding)
__device__ __forceinline__ double word_elem(uint32_t w, int e, const __nv_bfloat16*) {
    return (double)__uint_as_float(e == 0 ? w << 16 : w & 0xFFFF0000u);
}
__device__ __forceinline__ double word_elem(uint32_t w, int, const float*) { return (double)__uint_as_float(w); }

// acc + a_h * b_h for the bf16 values in the low (h = 0) / high (h = 1) halves
// of a and b: sm_100's mixed-precision fma, one rounding (the bf16 product is
// exact in fp32, so this equals fmaf on the widened values)
__device__ __forceinline__ float fma_bf16_lo(uint32_t a, uint32_t b, float acc) {
    float r;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %3;\n\t}" : "=f"(r) : "r"(a), "r"(b), "f"(acc));
    return r;
}
__device__ __forceinline__ float fma_bf16_hi(uint32_t a, uint32_t b, float acc) {
    float r;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %3;\n\t}" : "=f"(r) : "r"(a), "r"(b), "f"(acc));
    return r;
}
// k - c_h for the bf16 value c_h in the low / high half of w, rounded once
// (the mixed-precision fma c_h * -1 + k; identical to __fsub_rn on the
// widened value)
__device__ __forceinline__ float sub_bf16_lo(float k, uint32_t w) {
    float r;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tfma.rn.f32.bf16 %0, l, %2, %3;\n\t}"
        : "=f"(r) : "r"(w), "h"((unsigned short)0xBF80u), "f"(k));
    return r;
}
__device__ __forceinline__ float sub_bf16_hi(float k, uint32_t w) {
    float r;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tfma.rn.f32.bf16 %0, h, %2, %3;\n\t}"
        : "=f"(r) : "r"(w), "h"((unsigned short)0xBF80u), "f"(k));
    return r;
}

// One thread per key (a block: 128 keys of one (b,h)). The head's level-0
// rows are staged in shared memory (every thread of a warp reads the same row
// at the same time: broadcasts) and the key row is held in registers. Each
// step is decided on fp32 squared distances (fma(t, t) over t = fl(k - c),
// even and odd terms in two sums added at the end, whose error is bounded by
// dist_eps); where the bound cannot separate the winner from another
// candidate, the step is decided again on exact fp64 distances
// (exact_sq_dist: index order, no fusion) among the candidates it cannot
// separate, so that every decision is the exact one:
// level 0 the nearest node (first on ties), deeper levels a child only when
// strictly closer than the current node (first child on ties). The key's
// own node (the deepest on its path) counts it and sums its value row
// (16-byte vector reductions; the row was prefetched to L2 at the start);
// deep_totals_kernel then gives every node its whole subtree.
template <typename T, int D>
__global__ void __launch_bounds__(128)
deep_precompute_rows_kernel(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ cb,
                            int32_t* __restrict__ assign, int32_t* __restrict__ counts, float* __restrict__ vsum,
                            int N, int H, int ntiles, DeepTree t) {
    constexpr int EPW = 4 / (int)sizeof(T);     // elements per 32-bit word
    constexpr int U = D * (int)sizeof(T) / 16;  // 16-byte chunks per row
    extern __shared__ uint4 sC4[];              // [M0][U] the head's level-0 rows
    const int bh = blockIdx.x / ntiles, tile = blockIdx.x % ntiles, h = bh % H;
    const T* cbh = cb + (size_t)h * t.Mtot * D;
    for (int i = threadIdx.x; i < t.M0 * U; i += blockDim.x) sC4[i] = __ldg(reinterpret_cast<const uint4*>(cbh) + i);
    __syncthreads();
    const int n = tile * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const size_t key = (size_t)bh * N + n;
    {   // the value row is read after the descent: start bringing it to L2 now
        const char* vrow = reinterpret_cast<const char*>(V + key * D);
#pragma unroll
        for (int o = 0; o < D * (int)sizeof(T); o += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(vrow + o));
    }
    const T* tag = nullptr;
    // the key row, exact in fp32, as (even, odd) element pairs
    float2 kf[D / 2];
#pragma unroll
    for (int j = 0; j < U; ++j) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(K + key * D) + j);
        if constexpr (EPW == 2) {
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int w = 0; w < 4; ++w)
                kf[4 * j + w] = make_float2(__uint_as_float(w4[w] << 16), __uint_as_float(w4[w] & 0xFFFF0000u));
        } else {
            kf[2 * j] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
            kf[2 * j + 1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
        }
    }
    // fp32 squared distance to a row (shared or global memory): t = fl(k - c)
    // in one rounding, then fma(t, t) into an even-element and an odd-element
    // sum (sm_100 paired fp32 fma), added at the end -- two chains of d/2
    // terms, within the (d+2)u of dist_eps
    auto dist32 = [&](const uint4* row, bool shared) -> float {
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const uint4 u = shared ? row[j] : __ldg(row + j);
            if constexpr (EPW == 2) {
                const uint32_t cw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const float2 tt = make_float2(sub_bf16_lo(kf[4 * j + w].x, cw[w]),
                                                  sub_bf16_hi(kf[4 * j + w].y, cw[w]));
                    acc = __ffma2_rn(tt, tt, acc);
                }
            } else {
                const float2 m1 = make_float2(-1.f, -1.f);
                const float2 ta = __ffma2_rn(make_float2(__uint_as_float(u.x), __uint_as_float(u.y)), m1, kf[2 * j]);
                const float2 tb =
                    __ffma2_rn(make_float2(__uint_as_float(u.z), __uint_as_float(u.w)), m1, kf[2 * j + 1]);
                acc = __ffma2_rn(ta, ta, acc);
                acc = __ffma2_rn(tb, tb, acc);
            }
        }
        return __fadd_rn(acc.x, acc.y);
    };
    const float eps = dist_eps(D);
    const T* krow = K + key * D;
    auto row_of = [&](int r) { return reinterpret_cast<const uint4*>(cbh + (size_t)r * D); };
    // level 0: the nearest node
    float best = INFINITY, second = INFINITY;
    int bi = t.M0;
    for (int q = 0; q < t.M0; ++q) {
        const float dq = dist32(sC4 + (size_t)q * U, true);
        if (dq < best) {
            second = best;
            best = dq;
            bi = q;
        } else if (dq < second) {
            second = dq;
        }
    }
    if (t.M0 > 1 && !separated(best, second, eps)) {   // exact, among those the bound cannot separate
        double eb = INFINITY;
        int ep = -1;
        for (int q = 0; q < t.M0; ++q) {
            const float dq = dist32(sC4 + (size_t)q * U, true);
            if (separated(best, dq, eps)) continue;
            const double e = exact_sq_dist(krow, cbh + (size_t)q * D, D);
            if (e < eb) {
                eb = e;
                ep = q;
            }
        }
        if (ep >= 0) bi = ep;   // (ep < 0 only for non-finite inputs)
        best = dist32(sC4 + (size_t)(bi < t.M0 ? bi : 0) * U, true);
    }
    int local = bi < t.M0 ? bi : 0;   // (only non-finite inputs leave bi == M0)
    int node = local;
    for (int l = 1; l < t.L; ++l) {
        const int first = t.off[l] + local * t.C;
        // the current node first, then its children in index order; a child
        // wins only when strictly closer (the first kCh children's distances
        // stay in registers for the separation test)
        float lo = best;
        int ci = -1;
        float dch[kCh];
#pragma unroll
        for (int c = 0; c < kCh; ++c) {
            dch[c] = INFINITY;
            if (c < t.C) {
                dch[c] = dist32(row_of(first + c), false);
                if (dch[c] < lo) {
                    lo = dch[c];
                    ci = c;
                }
            }
        }
        for (int c = kCh; c < t.C; ++c) {
            const float dq = dist32(row_of(first + c), false);
            if (dq < lo) {
                lo = dq;
                ci = c;
            }
        }
        bool sure = ci < 0 || separated(lo, best, eps);
#pragma unroll
        for (int c = 0; c < kCh; ++c)
            if (c < t.C && c != ci && !separated(lo, dch[c], eps)) sure = false;
        for (int c = kCh; c < t.C && sure; ++c)
            if (c != ci && !separated(lo, dist32(row_of(first + c), false), eps)) sure = false;
        if (!sure) {   // exact, among the node and the children the bound cannot separate from the winner
            double eb = exact_sq_dist(krow, cbh + (size_t)node * D, D);
            int win = -1;
            for (int c = 0; c < t.C; ++c) {
                if (separated(lo, dist32(row_of(first + c), false), eps)) continue;
                const double e = exact_sq_dist(krow, cbh + (size_t)(first + c) * D, D);
                if (e < eb) {
                    eb = e;
                    win = c;
                }
            }
            ci = win;
            if (ci >= 0) lo = dist32(row_of(first + ci), false);
        }
        if (ci < 0) break;   // no child strictly closer: the descent stops
        best = lo;
        local = local * t.C + ci;
        node = first + ci;
    }
    const size_t base = (size_t)bh * t.Mtot;
    assign[key] = node;
    // the key's count and value row go to its own node only (the deepest on
    // its path); deep_totals_kernel then adds every node's subtree into it
    atomicAdd(counts + base + node, 1);
    // value row: four elements per reduction
#pragma unroll
    for (int j = 0; j < U; ++j) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(V + key * D) + j);
        const uint32_t vw[4] = {u.x, u.y, u.z, u.w};
        float f[4 * EPW];
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int e = 0; e < EPW; ++e) f[w * EPW + e] = (float)word_elem(vw[w], e, tag);
#pragma unroll
        for (int g = 0; g < EPW; ++g)
            red_add_v4(vsum + (base + node) * D + (size_t)j * 4 * EPW + 4 * g, f[4 * g], f[4 * g + 1], f[4 * g + 2],
                       f[4 * g + 3]);
    }
}

// One level of the subtree totals, launched from the deepest level with
// children upwards: each node of the level (width nodes from row `first`)
// adds its C children's counts and value sums, complete by then, to those of
// the keys that stopped at the node, so that it holds its whole subtree (the
// "every node on a key's path counts the key" rule). One thread per (node,
// 4 dimensions); the first of a node's threads also adds the counts.
__global__ void deep_totals_kernel(int32_t* __restrict__ counts, float* __restrict__ vsum, size_t BH, int Mtot,
                                   int first, int width, int child_first, int C, int d) {
    const int q = d / 4;   // 16-byte chunks of a row
    float4* v4 = reinterpret_cast<float4*>(vsum);
    const size_t n = BH * (size_t)width * q;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n; idx += (size_t)gridDim.x * blockDim.x) {
        const int k = (int)(idx % q);
        const size_t nd = idx / q;
        const int j = (int)(nd % width);
        const size_t bh = nd / width;
        const size_t row = bh * Mtot + first + j;
        const size_t crow = bh * Mtot + child_first + (size_t)j * C;
        float4 acc = v4[row * q + k];
        int cn = 0;
        for (int c = 0; c < C; ++c) {
            const float4 v = v4[(crow + c) * q + k];
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
            if (k == 0) cn += counts[crow + c];
        }
        v4[row * q + k] = acc;
        if (k == 0) counts[row] += cn;
    }
}

// fp32 value means vsum / n (0 for empty nodes)
__global__ void deep_means_kernel(const float* __restrict__ vsum, const int32_t* __restrict__ counts,
                                  float* __restrict__ mean, size_t rows, int d) {
    const size_t n = rows * (size_t)d;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int c = __ldg(counts + i / d);
        mean[i] = c > 0 ? __ldg(vsum + i) / (float)c : 0.f;
    }
}

struct DeepAttnArgs {
    const void* Q;
    const void* cb;
    const int32_t* counts;
    const float* mean;     // [BH, Mtot, D] fp32 means
    void* O;
    int32_t* selected;     // [BH, ntiles, sum_l P_l], level after level
    int N, H, ntiles, Psum;
    int ap_words;          // words of the Ap table: (largest P) rows of KT + 1, rounded up to 4
    int P[kMaxL];
    float sl2;             // scale * log2(e)
    DeepTree t;
};

// One CTA of KT threads per query tile, thread r owns query row r. Shared
// memory (padded strides keep both the per-row and the per-candidate access
// patterns free of bank conflicts):
//   Qs   [D][KT]            the tile's queries as fp32, transposed
//   E    [KC][KT + 1]       e'_c = A_c n_c of the current candidates per row
//   Ap   [Pmax][KT + 1]     A_f of the expanded candidates (by rank) per row
//   W    [KC]               importance of the current candidates
//   lgn  [KC]               log2 of the current candidates' counts
//   cid  [KC]               candidate row ids;  par [KC]: rank of a
//                           candidate's expanded parent;  sel [KC]: the
//                           expanded candidates (indices) by rank
//   Zs   [KT]               1 / Zbar per row (0 for rows past the end)
//   ncs  [KC]               counts of the current candidates
//   Cw   [KC][D]            the current candidates' codewords (raw T rows)
//   Mn   [KC][D]            their value means (fp32)
// At d = 64 the row's query is held in registers instead of Qs (bf16: packed,
// its logits by mixed-precision fma on the packed words). With ST the
// candidates' rows are staged once per level (Cw, Mn), so that the
// per-candidate loop reads shared-memory broadcasts; without (when they would
// not fit) it reads them from global memory, 16 bytes at a time. The
// candidate loops are unrolled four ways (more shared-memory reads in
// flight); for bf16 at d = 64 the launch bound keeps that within the
// registers of three CTAs per SM.
template <typename T, int D, int KT, int KC, bool ST>
__global__ void __launch_bounds__(KT, (D == 64 && sizeof(T) == 2) ? 3 : 1)
deep_attention_kernel(const DeepAttnArgs a) {
    extern __shared__ float sm[];
    constexpr int ES = KT + 1;
    const DeepTree& t = a.t;
    const int g = blockIdx.x, bh = g / a.ntiles, tt = g % a.ntiles, h = bh % a.H;
    const int r = threadIdx.x;
    const int i = tt * KT + r;
    const bool valid = i < a.N;
    constexpr bool QREG = D <= 64;                   // the query row in registers
    constexpr int CU = D * (int)sizeof(T) / 16;      // 16-byte chunks of a codeword row
    constexpr int MU = D / 4;                        // 16-byte chunks of a mean row
    float* Qs = sm;                                  // [D][KT] (unless QREG)
    float* E = Qs + (QREG ? 0 : D * KT);             // [KC][ES]
    float* Ap = E + KC * ES;                         // [Pmax][ES]
    float* W = Ap + a.ap_words;                      // [KC]
    float* Zs = W + KC;                              // [KT]
    float* lgn = Zs + KT;                            // [KC]
    int* cid = reinterpret_cast<int*>(lgn + KC);     // [KC]
    int* par = cid + KC;                             // [KC]
    int* sel = par + KC;                             // [KC]
    int* ncs = sel + KC;                             // [KC]
    uint4* Cw = reinterpret_cast<uint4*>(ncs + KC);  // [KC][CU] (16-byte aligned: every array above is a multiple of 4 words)
    float4* Mn = reinterpret_cast<float4*>(Cw + KC * CU);   // [KC][MU]
    const T* Q = static_cast<const T*>(a.Q);
    const T* cbh = static_cast<const T*>(a.cb) + (size_t)h * t.Mtot * D;
    const int32_t* cnt = a.counts + (size_t)bh * t.Mtot;
    const float* mn = a.mean + (size_t)bh * t.Mtot * D;

    const T* tag = nullptr;
    constexpr int EPV = 16 / (int)sizeof(T);   // elements per 16 bytes
    constexpr int EPW = 4 / (int)sizeof(T);    // elements per 32-bit word
    constexpr bool QPK = QREG && EPW == 2;           // bf16 row kept packed, two values per word
    float qv[(QREG && !QPK) ? D : 1];
    uint32_t qp[QPK ? D / 2 : 1];
    if constexpr (QREG) {   // this row's query
        const uint4* q4 = reinterpret_cast<const uint4*>(Q + ((size_t)bh * a.N + (valid ? i : 0)) * D);
#pragma unroll
        for (int v = 0; v < CU; ++v) {
            const uint4 u = valid ? __ldg(q4 + v) : make_uint4(0, 0, 0, 0);
            const uint32_t qw[4] = {u.x, u.y, u.z, u.w};
            if constexpr (QPK) {
#pragma unroll
                for (int w = 0; w < 4; ++w) qp[QPK ? 4 * v + w : 0] = qw[w];
            } else {
#pragma unroll
                for (int e = 0; e < EPV; ++e) qv[QPK ? 0 : v * EPV + e] = (float)word_elem(qw[e / EPW], e % EPW, tag);
            }
        }
    } else {   // the tile's queries, transposed (coalesced reads of whole rows)
        for (int idx = r; idx < KT * D; idx += KT) {
            const int rr = idx / D, j = idx % D;
            const int ii = tt * KT + rr;
            Qs[j * KT + rr] = ii < a.N ? ld_f32(Q + ((size_t)bh * a.N + ii) * D + j) : 0.f;
        }
    }
    // the nc current candidates' rows (ids in cid), counts, codewords and
    // value means, into shared memory (every thread; ends at a CTA barrier)
    auto stage = [&](int nc) {
        if constexpr (ST) {
            for (int idx = r; idx < nc * CU; idx += KT)
                Cw[idx] = __ldg(reinterpret_cast<const uint4*>(cbh + (size_t)cid[idx / CU] * D) + idx % CU);
            for (int idx = r; idx < nc * MU; idx += KT)
                Mn[idx] = __ldg(reinterpret_cast<const float4*>(mn + (size_t)cid[idx / MU] * D) + idx % MU);
        }
        for (int c = r; c < nc; c += KT) {
            const int n = __ldg(cnt + cid[c]);
            ncs[c] = n;
            lgn[c] = n > 0 ? __log2f((float)n) : -INFINITY;
        }
        __syncthreads();
    };
    // Q_i . codeword of candidate slot sl, fp32, in four interleaved sums
    auto logit = [&](int sl) -> float {
        const uint4* c4 = ST ? Cw + sl * CU : reinterpret_cast<const uint4*>(cbh + (size_t)cid[sl] * D);
        float s4[4] = {0.f, 0.f, 0.f, 0.f};   // element j goes to sum j % 4
#pragma unroll
        for (int v = 0; v < CU; ++v) {
            const uint4 u = ST ? c4[v] : __ldg(c4 + v);
            const uint32_t cw[4] = {u.x, u.y, u.z, u.w};
            if constexpr (QPK) {   // element 8v + 2w + h is word w's half h
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    s4[(2 * w) % 4] = fma_bf16_lo(qp[QPK ? 4 * v + w : 0], cw[w], s4[(2 * w) % 4]);
                    s4[(2 * w + 1) % 4] = fma_bf16_hi(qp[QPK ? 4 * v + w : 0], cw[w], s4[(2 * w + 1) % 4]);
                }
            } else {
#pragma unroll
                for (int e = 0; e < EPV; ++e) {
                    const int j = v * EPV + e;
                    const float qj = QREG ? qv[QREG ? j : 0] : Qs[j * KT + r];
                    s4[j % 4] = fmaf(qj, (float)word_elem(cw[e / EPW], e % EPW, tag), s4[j % 4]);
                }
            }
        }
        return (s4[0] + s4[1]) + (s4[2] + s4[3]);
    };
    // x += w * the value mean of candidate slot sl
    auto add_mean = [&](float (&xx)[D], float w, int sl) {
        const float4* m4 = ST ? Mn + sl * MU : reinterpret_cast<const float4*>(mn + (size_t)cid[sl] * D);
#pragma unroll
        for (int v = 0; v < D / 4; ++v) {
            const float4 q4 = ST ? m4[v] : __ldg(m4 + v);
            xx[4 * v] = fmaf(w, q4.x, xx[4 * v]);
            xx[4 * v + 1] = fmaf(w, q4.y, xx[4 * v + 1]);
            xx[4 * v + 2] = fmaf(w, q4.z, xx[4 * v + 2]);
            xx[4 * v + 3] = fmaf(w, q4.w, xx[4 * v + 3]);
        }
    };

    float x[D];
#pragma unroll
    for (int j = 0; j < D; ++j) x[j] = 0.f;
    // level 0: log-count logits, the row's shift m, weights e' = 2^(x - m)
    int ncand = t.M0;
    for (int c = r; c < ncand; c += KT) cid[c] = c;
    __syncthreads();
    stage(ncand);
    float m = -INFINITY;
#pragma unroll 4
    for (int c = 0; c < ncand; ++c) {
        const int n = ncs[c];
        const float xv = n > 0 ? fmaf(logit(c), a.sl2, lgn[c]) : -INFINITY;
        E[c * ES + r] = xv;
        m = fmaxf(m, xv);
    }
    float z = 0.f;
#pragma unroll 4
    for (int c = 0; c < ncand; ++c) {
        const float e = exp2f(E[c * ES + r] - m);   // 0 for empty nodes
        E[c * ES + r] = e;
        z += e;
        add_mean(x, e, c);
    }
    int soff = 0;
    for (int l = 0; l + 1 < t.L; ++l) {
        Zs[r] = valid && z > 0.f ? 1.f / z : 0.f;
        __syncthreads();
        // importance: sum over the tile's rows of e' / Zbar (Zbar so far), as
        // e' times the row's 1 / Zbar (0 for rows past the end)
        for (int c = r; c < ncand; c += KT) {
            float w0 = 0.f, w1 = 0.f;
#pragma unroll 4
            for (int rr = 0; rr < KT; rr += 2) {
                w0 = fmaf(E[c * ES + rr], Zs[rr], w0);
                w1 = fmaf(E[c * ES + rr + 1], Zs[rr + 1], w1);
            }
            W[c] = w0 + w1;
        }
        __syncthreads();
        const int P = min(a.P[l], ncand);
        // rank: larger importance first, ties to the lower row id
        for (int c = r; c < ncand; c += KT) {
            int rank = 0;
            const float wc = W[c];
            const int ic = cid[c];
            for (int q = 0; q < ncand; ++q) rank += (W[q] > wc) || (W[q] == wc && cid[q] < ic);
            if (rank < P) {
                sel[rank] = c;
                a.selected[((size_t)bh * a.ntiles + tt) * a.Psum + soff + rank] = ic;
            }
        }
        __syncthreads();
        // A_f = e'_f / n_f of the expanded candidates, kept while the
        // candidates are replaced by their children
        for (int k = 0; k < P; ++k) {
            const int c = sel[k];
            const int n = ncs[c];
            Ap[k * ES + r] = n > 0 ? E[c * ES + r] / (float)n : 0.f;
        }
        __syncthreads();   // every row has read the expanded candidates' ids and weights
        // the next candidates: the children of the expanded ones, in rank order
        int nid[KC / 32 + 1];
        int nn = 0;
        for (int s = r; s < P * t.C; s += KT) nid[nn++] = t.off[l + 1] + (cid[sel[s / t.C]] - t.off[l]) * t.C + s % t.C;
        __syncthreads();
        nn = 0;
        for (int s = r; s < P * t.C; s += KT) {
            cid[s] = nid[nn++];
            par[s] = s / t.C;
        }
        __syncthreads();
        ncand = P * t.C;
        stage(ncand);
        // pass 1: every candidate's exponent u = sl2 S + log2 n - m and the
        // largest one (the candidates are independent: unrolled for overlap)
        float umax = -INFINITY;
#pragma unroll 4
        for (int c = 0; c < ncand; ++c) {
            const int n = ncs[c];
            const float u = n > 0 ? fmaf(logit(c), a.sl2, lgn[c]) - m : -INFINITY;
            E[c * ES + r] = u;
            umax = fmaxf(umax, u);
        }
        float ku = 0.f;
        if (umax > kRescale) {
            // a child far above the row's shift: move the shift up by a whole
            // number k of octaves and scale everything this row holds by 2^-k
            // (exact), so that no weight overflows
            ku = ceilf(umax);
            const float f = exp2f(-ku);
            m += ku;
            z *= f;
#pragma unroll
            for (int j = 0; j < D; ++j) x[j] *= f;
            for (int kk = 0; kk < P; ++kk) Ap[kk * ES + r] *= f;
        }
        // pass 2: weights e' = 2^u, the corrections (A_g - A_f) n_g into Zbar
        // and Xbar
#pragma unroll 4
        for (int c = 0; c < ncand; ++c) {
            const int n = ncs[c];
            float e = 0.f;
            if (n > 0) {
                e = exp2f(E[c * ES + r] - ku);
                const float dw = e - Ap[par[c] * ES + r] * (float)n;   // (A_g - A_f) n_g
                z += dw;
                add_mean(x, dw, c);
            }
            E[c * ES + r] = e;
        }
        soff += a.P[l];
        __syncthreads();
    }
    if (valid) {
        const float inv = 1.f / z;
        T* o = static_cast<T*>(a.O) + ((size_t)bh * a.N + i) * D;
#pragma unroll
        for (int j = 0; j < D; ++j) st_elem(o + j, x[j] * inv);
    }
}

// words of the Ap table: one row of KT + 1 per expanded candidate of the
// level that expands the most, rounded up to 4 (keeps the arrays after it
// 16-byte aligned)
int deep_ap_words(const DeepAttnArgs& a, int KT) {
    int pmax = 0;
    for (int l = 0; l + 1 < a.t.L; ++l) pmax = std::max(pmax, a.P[l]);
    return (pmax * (KT + 1) + 3) & ~3;
}
size_t deep_attn_smem(int D, int KT, int KC, size_t elem, bool staged, int ap_words) {
    const size_t qs = D <= 64 ? 0 : (size_t)D * KT;   // (the query rows are in registers at d <= 64)
    return sizeof(float) * (qs + (size_t)KC * (KT + 1) + (size_t)ap_words + 2 * KC + KT) + sizeof(int) * 4 * KC +
           (staged ? (size_t)KC * D * (elem + sizeof(float)) : 0);
}

template <typename T, int D>
cudaError_t launch_deep_pre(const avq_shape& s, const DeepTree& t, const void* K, const void* V, const void* cb,
                            int32_t* assign, int32_t* counts, float* vsum, cudaStream_t st) {
    const int ntiles = (s.N + 127) / 128;
    const size_t smem = (size_t)t.M0 * D * sizeof(T);
    auto kern = deep_precompute_rows_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)((long long)s.B * s.H * ntiles), 128, smem, st>>>(
        static_cast<const T*>(K), static_cast<const T*>(V), static_cast<const T*>(cb), assign, counts, vsum, s.N, s.H,
        ntiles, t);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t BH = (size_t)s.B * s.H;
    for (int l = t.L - 2; l >= 0; --l) {
        const int width = t.off[l + 1] - t.off[l];
        const size_t n = BH * (size_t)width * (D / 4);
        deep_totals_kernel<<<(unsigned)std::min<size_t>((n + 255) / 256, 4096), 256, 0, st>>>(
            counts, vsum, BH, t.Mtot, t.off[l], width, t.off[l + 1], t.C, D);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <typename T, int D, int KT, int KC>
cudaError_t launch_deep_att(DeepAttnArgs a, int tiles, cudaStream_t st) {
    a.ap_words = deep_ap_words(a, KT);
    // the candidates' rows staged in shared memory when the CTA still fits
    const bool staged = deep_attn_smem(D, KT, KC, sizeof(T), true, a.ap_words) <= 227 * 1024;
    const size_t smem = deep_attn_smem(D, KT, KC, sizeof(T), staged, a.ap_words);
    auto kern = staged ? deep_attention_kernel<T, D, KT, KC, true> : deep_attention_kernel<T, D, KT, KC, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)tiles, KT, smem, st>>>(a);
    count_launch();
    return cudaGetLastError();
}

int check_deep(const avq_shape* s, int L) {
    int rc = check_shape(s);
    if (rc != AVQ_OK) return rc;
    if (L < 2 || L > kMaxL || s->C < 1) return AVQ_EINVAL;
    if (s->M0 > kCand) return AVQ_EUNSUPPORTED;
    if (deep_rows(s->M0, s->C, L) >= (1LL << 24)) return AVQ_EUNSUPPORTED;
    if ((long long)s->B * s->H * deep_rows(s->M0, s->C, L) * s->d >= (1LL << 40)) return AVQ_EUNSUPPORTED;
    return AVQ_OK;
}

bool aligned_p(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace avq

using namespace avq;

extern "C" {

int avq_precompute_deep(const avq_shape* s, int L, const void* K, const void* V, const void* codebook,
                        int32_t* assign, int32_t* counts, float* vsum, void* stream) {
    int rc = check_deep(s, L);
    if (rc != AVQ_OK) return rc;
    if (!codebook || !counts || !vsum) return AVQ_EINVAL;
    if (s->N > 0 && (!K || !V || !assign)) return AVQ_EINVAL;
    if (!aligned_p(K, 16) || !aligned_p(V, 16) || !aligned_p(codebook, 16) || !aligned_p(vsum, 16) ||
        !aligned_p(assign, 4) || !aligned_p(counts, 4))
        return AVQ_EINVAL;
    const DeepTree t = make_tree(s->M0, s->C, L);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t BH = (size_t)s->B * s->H;
    if (cudaMemsetAsync(counts, 0, BH * t.Mtot * sizeof(int32_t), st) != cudaSuccess) return AVQ_ECUDA;
    if (cudaMemsetAsync(vsum, 0, BH * t.Mtot * s->d * sizeof(float), st) != cudaSuccess) return AVQ_ECUDA;
    if (s->N == 0) return AVQ_OK;
    cudaError_t e;
    if (s->dtype == AVQ_BF16)
        e = s->d == 64 ? launch_deep_pre<__nv_bfloat16, 64>(*s, t, K, V, codebook, assign, counts, vsum, st)
                       : launch_deep_pre<__nv_bfloat16, 128>(*s, t, K, V, codebook, assign, counts, vsum, st);
    else
        e = s->d == 64 ? launch_deep_pre<float, 64>(*s, t, K, V, codebook, assign, counts, vsum, st)
                       : launch_deep_pre<float, 128>(*s, t, K, V, codebook, assign, counts, vsum, st);
    return e == cudaSuccess ? AVQ_OK : AVQ_ECUDA;
}

size_t avq_attention_deep_workspace_bytes(const avq_shape* s, int L) {
    if (check_deep(s, L) != AVQ_OK) return 0;
    return kStatusBytes + align256((size_t)s->B * s->H * deep_rows(s->M0, s->C, L) * s->d * sizeof(float));
}

int avq_attention_deep(const avq_shape* s, int L, const int32_t* P, const void* Q, const void* codebook,
                       const int32_t* counts, const float* vsum, int tile, float scale, void* O, int32_t* selected,
                       void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_deep(s, L);
    if (rc != AVQ_OK) return rc;
    if (!P || (tile != 64 && tile != 128)) return AVQ_EINVAL;
    if (!(scale > 0.f) || !(scale < 3.0e38f)) return AVQ_EINVAL;
    DeepAttnArgs a{};
    a.t = make_tree(s->M0, s->C, L);
    a.Psum = 0;
    for (int l = 0; l + 1 < L; ++l) {
        const long long ncand = l == 0 ? s->M0 : (long long)P[l - 1] * s->C;
        if (P[l] < 0 || P[l] > ncand || (long long)P[l] * s->C > kCand) return AVQ_EINVAL;
        a.P[l] = P[l];
        a.Psum += P[l];
    }
    if (!codebook || !counts || !vsum) return AVQ_EINVAL;
    if (s->N > 0 && (!Q || !O || (a.Psum > 0 && !selected))) return AVQ_EINVAL;
    if (!aligned_p(Q, 16) || !aligned_p(O, 16) || !aligned_p(codebook, 16) || !aligned_p(vsum, 16) ||
        !aligned_p(counts, 4) || !aligned_p(selected, 4))
        return AVQ_EINVAL;
    const size_t need = avq_attention_deep_workspace_bytes(s, L);
    if (!workspace || workspace_bytes < need) return AVQ_EWORKSPACE;
    if (!aligned_p(workspace, 256)) return AVQ_EINVAL;
    if (s->N == 0) return AVQ_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* means = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kStatusBytes);
    const size_t rows = (size_t)s->B * s->H * a.t.Mtot;
    deep_means_kernel<<<(unsigned)std::min<size_t>((rows * s->d + 255) / 256, 4096), 256, 0, st>>>(vsum, counts,
                                                                                                    means, rows, s->d);
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return AVQ_ECUDA;
    a.Q = Q;
    a.cb = codebook;
    a.counts = counts;
    a.mean = means;
    a.O = O;
    a.selected = selected;
    a.N = s->N;
    a.H = s->H;
    a.ntiles = (s->N + tile - 1) / tile;
    a.sl2 = scale * 1.4426950408889634f;
    const int tiles = s->B * s->H * a.ntiles;
    cudaError_t e = cudaErrorInvalidValue;   // (every supported d and tile has a case below)
    // candidates per level held on chip: 64 when no level has more (the
    // per-row tables halve: two CTAs per SM at d = 64 and 128-row tiles),
    // else 128
    int maxc = s->M0;
    for (int l = 0; l + 1 < L; ++l) maxc = std::max(maxc, a.P[l] * s->C);
    const bool kc64 = maxc <= 64;
#define AVQ_DEEP_CASE(TT, DD, KK)                                                                     \
    if (s->d == DD && tile == KK)                                                                     \
        e = kc64 ? launch_deep_att<TT, DD, KK, 64>(a, tiles, st) : launch_deep_att<TT, DD, KK, 128>(a, tiles, st);
    if (s->dtype == AVQ_BF16) {
        AVQ_DEEP_CASE(__nv_bfloat16, 64, 64) AVQ_DEEP_CASE(__nv_bfloat16, 64, 128)
        AVQ_DEEP_CASE(__nv_bfloat16, 128, 64) AVQ_DEEP_CASE(__nv_bfloat16, 128, 128)
    } else {
        AVQ_DEEP_CASE(float, 64, 64) AVQ_DEEP_CASE(float, 64, 128)
        AVQ_DEEP_CASE(float, 128, 64) AVQ_DEEP_CASE(float, 128, 128)
    }
#undef AVQ_DEEP_CASE
    return e == cudaSuccess ? AVQ_OK : AVQ_ECUDA;
}

}  // extern "C"
