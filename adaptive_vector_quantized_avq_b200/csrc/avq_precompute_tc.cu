// avq_precompute_tc.cu -- tensor-core (tcgen05) kernel of avq_precompute for
// bf16 inputs (paper §4.2; papernotes, Key Designs 2; paper Table 1 rows
// "VQ assignment" and "Value aggregation").
//
// Persistent: one 256-thread CTA per SM walks a contiguous range of 128-key
// tiles (head-major). Key r of a tile is handled by the thread pair r and
// r + 128 (halves h = 0, 1): each half holds half of the key's dimensions and
// scans half of the parents. The pair combines its parent scans through shared
// memory (both threads then hold the same nearest parent); for the children,
// half 1 publishes its partial distances and half 0 completes them, decides
// and writes the outputs. TMEM lane r holds key r's dot products.
//
// Per head (when the range enters it): TMA brings the parent codewords (the
// B operand), cp.async brings the C*M0 child codewords into a shared-memory
// image whose 16-byte chunks are permuted by the parent index (so that keys
// of different parents read different banks), and the parent norms
// ||C_p||^2 are computed. Counts accumulate in shared memory and are flushed
// with one global atomic per non-empty codeword when the head is done.
//
// Per tile:
//   1. TMA brings K and V (two stages, issued two tiles ahead).
//   2. MMA  S = K C_par^T  (M=128, N=M0p, K=d) into one of two TMEM buffers,
//      issued one tile ahead.
//   3. a1: v_p = ||C_p||^2 - 2 S_p (the expanded distance minus ||k||^2) in
//      fp32; the smallest and the runner-up. If they are not separated by the
//      error bound of this expanded form, the parents within the band are
//      re-decided with the exact fp64 distance summed in index order.
//   4. a2: the kept parent and its C children by the direct form
//      sum_j (k_j - c_j)^2 in fp32 (sm_100 mixed bf16/fp32 subtraction, so
//      the codewords need no unpacking; relative error <= (d+4)u); a
//      candidate wins only when strictly closer (parent first,
//      lowest child index among equals); the band the bound cannot separate
//      is re-decided in fp64.
//   5. a3: assign written; counts in shared memory; the key's V row is added
//      to the parent's and (when the key moved) the child's value sum with
//      coalesced 16-byte fp32 vector reductions (one half-warp per row).
#include <algorithm>

#include "avq_internal.cuh"
#include "avq_sm100.cuh"

namespace avq {
using namespace sm100;

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr uint32_t kRegion = 128 * 128;

struct TcPreParams {
    int BH, H, N, M0, M0p, Mtot, ntiles, total_tiles;
    const uint16_t* K;          // [BH, N, D] bf16 (exact re-decisions read keys here)
    const uint16_t* codebook;   // [H, Mtot, D] bf16
    int32_t* assign;            // [BH, N]
    int32_t* counts;            // [BH, Mtot]
    float* vsum;                // [BH, Mtot, D]
    StatusBlock* status;
};

__device__ __forceinline__ uint8_t* align1024p(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
// K-major operand, k-step ks, of a [rows x D] bf16 image whose 64-column
// blocks are `region` bytes apart
__device__ __forceinline__ uint64_t desc_k128(const uint8_t* img, int ks, uint32_t region = kRegion) {
    const uint32_t a = smem_u32(img) + (uint32_t)(ks >> 2) * region + (uint32_t)(ks & 3) * 32u;
    return smem_desc_sw128(a, 16, 1024);
}
// 16-byte chunk j of row r of a TMA 128-byte-swizzled [rows x D] image
__device__ __forceinline__ uint32_t swz_off(int r, int j, uint32_t region = kRegion) {
    return (uint32_t)(j >> 3) * region + (uint32_t)r * 128u + (uint32_t)(((j & 7) ^ (r & 7)) << 4);
}
// 16-byte chunk j of child row i (parent p = i / C) in the children image
template <int D>
__device__ __forceinline__ uint32_t ch_off(int i, int p, int j) {
    return (uint32_t)i * (D * 2) + (uint32_t)(((j & ~7) | ((j & 7) ^ (p & 7))) << 4);
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// (c - k) for a bf16 c (low or high half of a 32-bit word) and an fp32 k,
// rounded once (sm_100 mixed-precision subtraction; no unpacking)
__device__ __forceinline__ float sub_lo(uint32_t w, float k) {
    float r;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tsub.rn.f32.bf16 %0, l, %2;\n\t}" : "=f"(r) : "r"(w), "f"(k));
    return r;
}
__device__ __forceinline__ float sub_hi(uint32_t w, float k) {
    float r;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tsub.rn.f32.bf16 %0, h, %2;\n\t}" : "=f"(r) : "r"(w), "f"(k));
    return r;
}

// Partial squared distance over this half's NC 16-byte chunks (chunk index
// offset j0) of the key (fp32) to a bf16 row in shared memory whose chunk j
// lives at chunk_off(j); each term (k - c)^2 rounded once (fused), four
// independent accumulators.
template <int NC, typename F>
__device__ __forceinline__ float half_dist(const float (&k)[NC * 8], const uint8_t* row_base, int j0,
                                           F chunk_off) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        const uint4 w = *reinterpret_cast<const uint4*>(row_base + chunk_off(j0 + j));
        const float t0 = sub_lo(w.x, k[8 * j + 0]), t1 = sub_hi(w.x, k[8 * j + 1]);
        const float t2 = sub_lo(w.y, k[8 * j + 2]), t3 = sub_hi(w.y, k[8 * j + 3]);
        const float t4 = sub_lo(w.z, k[8 * j + 4]), t5 = sub_hi(w.z, k[8 * j + 5]);
        const float t6 = sub_lo(w.w, k[8 * j + 6]), t7 = sub_hi(w.w, k[8 * j + 7]);
        a0 = __fmaf_rn(t0, t0, a0); a1 = __fmaf_rn(t1, t1, a1);
        a2 = __fmaf_rn(t2, t2, a2); a3 = __fmaf_rn(t3, t3, a3);
        a0 = __fmaf_rn(t4, t4, a0); a1 = __fmaf_rn(t5, t5, a1);
        a2 = __fmaf_rn(t6, t6, a2); a3 = __fmaf_rn(t7, t7, a3);
    }
    return __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
}

// Exact fp64 distance between two global bf16 rows, terms in index order,
// no fused operations.
template <int D>
__device__ __noinline__ double exact_dist_glob(const uint16_t* k, const uint16_t* c) {
    double s = 0.0;
    for (int j = 0; j < D; ++j) {
        const double kj = (double)__uint_as_float((uint32_t)__ldg(k + j) << 16);
        const double cj = (double)__uint_as_float((uint32_t)__ldg(c + j) << 16);
        const double t = __dsub_rn(kj, cj);
        s = __dadd_rn(s, __dmul_rn(t, t));
    }
    return s;
}

__device__ __forceinline__ void red_v2(float* addr, float a, float b) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(addr), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void red_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

template <int D, int C, int KVS>
__global__ void __launch_bounds__(kThreads, 1)
precompute_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmCB, const TcPreParams p) {
    constexpr int KH = D / 64;
    constexpr uint32_t IMG = KH * kRegion;
    constexpr int KSTEPS = D / 16;
    constexpr int NCH = D / 16;          // 16-byte chunks per half row
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align1024p(smem_raw);
    uint8_t* sK0 = base;                     // K stages: sK0 + s*IMG (KVS of them)
    uint8_t* sV0 = base + KVS * IMG;         // V stages
    uint8_t* sB1 = base + 2 * KVS * IMG;     // parent codewords (K-major, TMA), M0p rows
    const uint32_t b1_region = (uint32_t)p.M0p * 128u;   // bytes between its 64-column blocks
    uint8_t* sCh = sB1 + KH * b1_region;     // children image [M0*C rows x D] bf16
    const size_t ch_bytes = (size_t)p.M0 * C * D * 2;
    float* sCn = reinterpret_cast<float*>(sCh + ((ch_bytes + 15) & ~size_t(15)));   // [128]
    float* sKn = sCn + 128;                  // [2][128] partial ||k||^2
    float* sBest = sKn + 256;                // [2][128]
    float* sSecond = sBest + 256;            // [2][128]
    int* sIdx = reinterpret_cast<int*>(sSecond + 256);       // [2][128]
    float* sDist = reinterpret_cast<float*>(sIdx + 256);     // [C+1][128] partial distances of half 1
    int* sPar = reinterpret_cast<int*>(sDist + (C + 1) * 128);       // [128]
    int* sLeaf = sPar + 128;                 // [128]
    float* sRed = reinterpret_cast<float*>(sLeaf + 128);     // [8]
    int* sCnt = reinterpret_cast<int*>(sRed + 8);            // [Mtot]
    uint64_t* bars = reinterpret_cast<uint64_t*>(
        (reinterpret_cast<uintptr_t>(sCnt + p.Mtot) + 7) & ~uintptr_t(7));
    // bars: 0,1 = K stage; 2,3 = V stage; 4,5 = MMA buffer; 6 = head
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 7);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = tid & 127, half = tid >> 7;
    const int g0 = (int)(((long long)blockIdx.x * p.total_tiles) / gridDim.x);
    const int g1 = (int)(((long long)(blockIdx.x + 1) * p.total_tiles) / gridDim.x);

    if (warp == 0) {
        tmem_alloc(sTmem, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 7; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmCB);
    }
    for (int i = tid; i < p.Mtot; i += kThreads) sCnt[i] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t idesc = idesc_bf16_f32(128, p.M0p, false);
    const float eps_dir = dist_eps(D);
    // expanded-form bound factor: 2 * (5d + 8) * 2^-24 (per distance, times
    // ||k||^2 + max ||C_p||^2)
    const float c_exp = 2.f * (5.f * D + 8.f) * 5.9604644775390625e-08f;

    uint32_t kph = 0, vph = 0, mph = 0, hph = 0;   // phase bit of stage s = bit s
    bool failed = false;
    int cur_bh = -1;
    float cnmax = 0.f;
    int n_pre = 0, n_chd = 0;   // fp64 re-decisions (diagnostics)

    auto issue_kv = [&](int g, int s) {   // K and V tiles of tile g into stage s
        const int bh = g / p.ntiles, t = g % p.ntiles;
        mbar_arrive_expect_tx(&bars[s], IMG);
        mbar_arrive_expect_tx(&bars[2 + s], IMG);
#pragma unroll
        for (int kh = 0; kh < KH; ++kh) {
            tma_load_3d(sK0 + s * IMG + kh * kRegion, &tmK, &bars[s], kh * 64, t * kTile, bh);
            tma_load_3d(sV0 + s * IMG + kh * kRegion, &tmV, &bars[2 + s], kh * 64, t * kTile, bh);
        }
    };
    auto issue_mma = [&](int s, int tb) -> bool {   // tid 0 only: K stage s -> TMEM buffer tb
        const bool ok = mbar_wait(&bars[s], (kph >> s) & 1u);
        kph ^= 1u << s;
        if (!ok) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks)
            mma_ss(tmem + 128 * tb, desc_k128(sK0 + s * IMG, ks), desc_k128(sB1, ks, b1_region), idesc, ks > 0);
        mma_commit(&bars[4 + tb]);
        return true;
    };
    auto flush_counts = [&](int bh) {
        for (int i = tid; i < p.Mtot; i += kThreads) {
            const int c = sCnt[i];
            if (c) {
                atomicAdd(p.counts + (size_t)bh * p.Mtot + i, c);
                sCnt[i] = 0;
            }
        }
    };

    if (tid == 0 && g0 < g1) {
        issue_kv(g0, 0);
        if (KVS == 2 && g0 + 1 < g1) issue_kv(g0 + 1, 1);
    }
    bool mma_issued_ahead = false;   // MMA of the current tile already issued

    for (int g = g0, it = 0; g < g1; ++g, ++it) {
        const int s = KVS == 2 ? (it & 1) : 0;   // K/V stage
        const int tb = it & 1;                   // TMEM buffer of this tile's dot products
        const int bh = g / p.ntiles, t = g % p.ntiles, h = bh % p.H;
        const int rows = min(kTile, p.N - t * kTile);
        const bool valid = r < rows;

        if (bh != cur_bh) {
            // flush the previous head's counts, load the new head's codewords
            if (cur_bh >= 0) flush_counts(cur_bh);
            if (cur_bh < 0 || h != cur_bh % p.H) {
                if (tid == 0) {
                    mbar_arrive_expect_tx(&bars[6], KH * (uint32_t)p.M0p * 128u);
#pragma unroll
                    for (int kh = 0; kh < KH; ++kh) tma_load_3d(sB1 + kh * b1_region, &tmCB, &bars[6], kh * 64, 0, h);
                }
                const uint16_t* chg = p.codebook + ((size_t)h * p.Mtot + p.M0) * D;
                for (int idx = tid; idx < p.M0 * C * (D / 8); idx += kThreads) {
                    const int i = idx / (D / 8), j = idx % (D / 8);
                    cp_async_16(sCh + ch_off<D>(i, i / C, j), chg + (size_t)i * D + j * 8);
                }
                cp_async_commit();
                float cn = 0.f;
                if (tid < p.M0) {
                    const uint16_t* cp = p.codebook + ((size_t)h * p.Mtot + tid) * D;
#pragma unroll 8
                    for (int j = 0; j < D; ++j) {
                        const float c = __uint_as_float((uint32_t)__ldg(cp + j) << 16);
                        cn = __fmaf_rn(c, c, cn);
                    }
                }
                if (tid < 128) sCn[tid] = tid < p.M0 ? cn : INFINITY;
                float mx = cn;
#pragma unroll
                for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                if (lane == 0) sRed[warp] = mx;
                cp_async_wait_all();
                fence_proxy_async_smem();
                const bool ok = mbar_wait(&bars[6], hph);
                hph ^= 1;
                if (__syncthreads_or(!ok)) { failed = true; break; }
                cnmax = fmaxf(fmaxf(sRed[0], sRed[1]), fmaxf(sRed[2], sRed[3]));
                mma_issued_ahead = false;
            } else {
                __syncthreads();
            }
            cur_bh = bh;
        }

        bool ok = true;
        if (tid == 0 && !mma_issued_ahead) ok = issue_mma(s, tb);
        // (if thread 0 could not issue the MMA, every thread's wait below times out)
        ok = mbar_wait(&bars[4 + tb], (mph >> tb) & 1u) && ok;
        mph ^= 1u << tb;
        if (__syncthreads_or(!ok)) { failed = true; break; }
        tc_fence_after();

        // this half of the key row -> fp32; partial ||k||^2
        float k[NCH * 8];
        {
            const uint8_t* kimg = sK0 + s * IMG;
            float kn0 = 0.f, kn1 = 0.f;
#pragma unroll
            for (int j = 0; j < NCH; ++j) {
                const uint4 w = *reinterpret_cast<const uint4*>(kimg + swz_off(r, half * NCH + j));
                k[8 * j + 0] = bf_lo(w.x); k[8 * j + 1] = bf_hi(w.x);
                k[8 * j + 2] = bf_lo(w.y); k[8 * j + 3] = bf_hi(w.y);
                k[8 * j + 4] = bf_lo(w.z); k[8 * j + 5] = bf_hi(w.z);
                k[8 * j + 6] = bf_lo(w.w); k[8 * j + 7] = bf_hi(w.w);
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    kn0 = __fmaf_rn(k[8 * j + e], k[8 * j + e], kn0);
                    kn1 = __fmaf_rn(k[8 * j + e + 1], k[8 * j + e + 1], kn1);
                }
            }
            sKn[half * 128 + r] = __fadd_rn(kn0, kn1);
        }

        // issue the next tile's MMA into the other TMEM buffer (same head, and
        // only when its K tile is already on the way: two K/V stages)
        mma_issued_ahead = false;
        if (KVS == 2 && g + 1 < g1 && (g + 1) / p.ntiles == bh) {
            if (tid == 0) ok = issue_mma(s ^ 1, tb ^ 1);
            mma_issued_ahead = true;
        }

        // ---- a1: this half's parents (16-column chunks c with c % 2 == half);
        // four independent trackers over interleaved columns, merged at the end
        {
            float best[4], second[4];
            int bp[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) { best[u] = INFINITY; second[u] = INFINITY; bp[u] = 0x7fffffff; }
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int c = 2 * cc + half;
                if (16 * c < p.M0p) {
                    uint32_t v16[16];
                    tmem_ld16(trow + 128 * tb + 16 * c, v16);
                    tmem_wait_ld();
                    tmem_touch16(v16);
#pragma unroll
                    for (int q = 0; q < 16; q += 4) {
                        // ||C_p||^2 is +inf for padding parents (p >= M0)
                        const float4 cn4 = *reinterpret_cast<const float4*>(sCn + 16 * c + q);
                        const float cnq[4] = {cn4.x, cn4.y, cn4.z, cn4.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int pp = 16 * c + q + u;
                            const float v = fmaf(-2.f, __uint_as_float(v16[q + u]), cnq[u]);
                            if (v < best[u]) { second[u] = best[u]; best[u] = v; bp[u] = pp; }
                            else second[u] = fminf(second[u], v);
                        }
                    }
                }
            }
            // merge the four trackers (lowest index among equal values)
#pragma unroll
            for (int u = 1; u < 4; ++u) {
                const bool take = (best[u] < best[0]) || (best[u] == best[0] && bp[u] < bp[0]);
                const float lo = take ? best[u] : best[0], hi = take ? best[0] : best[u];
                second[0] = fminf(hi, fminf(second[0], second[u]));
                best[0] = lo;
                bp[0] = take ? bp[u] : bp[0];
            }
            sBest[half * 128 + r] = best[0];
            sSecond[half * 128 + r] = second[0];
            sIdx[half * 128 + r] = bp[0];
        }
        __syncthreads();
        const float kn = sKn[r] + sKn[128 + r];
        float best, second;
        int bp;
        {
            const float b0 = sBest[r], b1 = sBest[128 + r];
            const int i0 = sIdx[r], i1 = sIdx[128 + r];
            const bool take1 = (b1 < b0) || (b1 == b0 && i1 < i0);
            best = take1 ? b1 : b0;
            bp = take1 ? i1 : i0;
            second = fminf(fmaxf(b0, b1), fminf(sSecond[r], sSecond[128 + r]));
            if (bp >= p.M0) bp = 0;   // no parent column (cannot happen for M0 >= 1)
        }
        const uint16_t* cbh = p.codebook + (size_t)h * p.Mtot * D;
        const uint16_t* krow = p.K + ((size_t)bh * p.N + (size_t)t * kTile + r) * D;
        const float E = c_exp * (kn + cnmax);
        const bool redecide = valid && p.M0 > 1 && !(second - best > 2.f * E);
        if (__any_sync(0xffffffffu, redecide)) {
            // re-decide among the parents within the band, in fp64; both halves
            // do it and reach the same result. TMEM reloads are warp-wide.
            double eb = INFINITY;
            int ep = bp;
            for (int c = 0; c < p.M0p; c += 16) {
                uint32_t v16[16];
                tmem_ld16(trow + 128 * tb + c, v16);
                tmem_wait_ld();
                tmem_touch16(v16);
                if (redecide) {
                    for (int q = 0; q < 16; ++q) {
                        const int pp = c + q;
                        if (pp >= p.M0) break;
                        const float v = fmaf(-2.f, __uint_as_float(v16[q]), sCn[pp]);
                        if (v - best > 2.f * E) continue;
                        const double e = exact_dist_glob<D>(krow, cbh + (size_t)pp * D);
                        if (e < eb) { eb = e; ep = pp; }
                    }
                }
            }
            if (redecide) {
                bp = ep;
                if (half == 0) ++n_pre;
            }
        }

        // ---- a2: partial direct distances of the kept parent and its children;
        // half 1 publishes its partials, half 0 completes them and decides
        float part[C + 1];
        part[0] = half_dist<NCH>(k, sB1, half * NCH, [&](int j) { return swz_off(bp, j, b1_region); });
#pragma unroll
        for (int c = 0; c < C; ++c) {
            const int i = bp * C + c;
            part[1 + c] = half_dist<NCH>(k, sCh, half * NCH, [&](int j) { return ch_off<D>(i, bp, j); });
        }
        if (half == 1) {
#pragma unroll
            for (int c = 0; c <= C; ++c) sDist[c * 128 + r] = part[c];
        }
        __syncthreads();
        int leaf = bp;
        if (half == 0) {
            const float dpar = __fadd_rn(part[0], sDist[r]);
            float dch[C];
            float lo = dpar;
            int lo_i = -1;
#pragma unroll
            for (int c = 0; c < C; ++c) {
                dch[c] = __fadd_rn(part[1 + c], sDist[(1 + c) * 128 + r]);
                if (dch[c] < lo) { lo = dch[c]; lo_i = c; }
            }
            bool sure = (lo_i < 0) || separated(lo, dpar, eps_dir);
#pragma unroll
            for (int c = 0; c < C; ++c)
                if (c != lo_i && !separated(lo, dch[c], eps_dir)) sure = false;
            if (sure || !valid) {
                leaf = lo_i < 0 ? bp : p.M0 + bp * C + lo_i;
            } else {
                double eb = exact_dist_glob<D>(krow, cbh + (size_t)bp * D);
                int win = bp;
#pragma unroll
                for (int c = 0; c < C; ++c) {
                    if (separated(lo, dch[c], eps_dir)) continue;
                    const double e = exact_dist_glob<D>(krow, cbh + (size_t)(p.M0 + bp * C + c) * D);
                    if (e < eb) { eb = e; win = p.M0 + bp * C + c; }
                }
                leaf = win;
                ++n_chd;
            }
        }

        // ---- a3: outputs
        if (half == 0) {
            if (valid) {
                p.assign[(size_t)bh * p.N + t * kTile + r] = leaf;
                atomicAdd(&sCnt[bp], 1);
                if (leaf != bp) atomicAdd(&sCnt[leaf], 1);
            }
            sPar[r] = valid ? bp : -1;
            sLeaf[r] = leaf;
        }
        const bool ok_v = mbar_wait(&bars[2 + s], (vph >> s) & 1u);
        vph ^= 1u << s;
        if (__syncthreads_or(!ok || !ok_v)) { failed = true; break; }   // also: K stage s no longer read

        // value sums: warp w adds the V rows of keys 16w..16w+15, two keys per
        // step (one per half-warp); lane l of a half holds 4 (d = 64) or 8
        // (d = 128) consecutive dimensions of the row
        {
            const uint8_t* vimg = sV0 + s * IMG;
            const int hl = lane & 15, sub = lane >> 4;
            constexpr int DPL = D / 16;                       // dimensions per lane
            const int j = (hl * DPL) >> 3;                    // 16-byte chunk of those dimensions
            const uint32_t inchunk = ((hl * DPL) & 7) * 2;    // byte offset inside the chunk
            float* vs_lane = p.vsum + (size_t)bh * p.Mtot * D + hl * DPL;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int rr = 16 * warp + 2 * q + sub;
                const int par = sPar[rr];
                const int lf = sLeaf[rr];
                if (par >= 0) {
                    const uint8_t* src = vimg + swz_off(rr, j) + inchunk;
                    if (D == 64) {
                        const uint2 w = *reinterpret_cast<const uint2*>(src);
                        const float a = bf_lo(w.x), b = bf_hi(w.x), c = bf_lo(w.y), d = bf_hi(w.y);
                        red_v4(vs_lane + (size_t)par * D, a, b, c, d);
                        if (lf != par) red_v4(vs_lane + (size_t)lf * D, a, b, c, d);
                    } else {
                        const uint4 w = *reinterpret_cast<const uint4*>(src);
                        red_v4(vs_lane + (size_t)par * D, bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
                        red_v4(vs_lane + (size_t)par * D + 4, bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w));
                        if (lf != par) {
                            red_v4(vs_lane + (size_t)lf * D, bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
                            red_v4(vs_lane + (size_t)lf * D + 4, bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w));
                        }
                    }
                }
            }
        }
        __syncthreads();
        if (tid == 0 && g + KVS < g1) issue_kv(g + KVS, s);
    }

    if (!failed && cur_bh >= 0) flush_counts(cur_bh);
    if (failed && tid == 0) {
        atomicExch(&p.status->error, (int)AVQ_ETIMEOUT);
        atomicExch(&p.status->where, (int)blockIdx.x);
    }
    if (n_pre) atomicAdd(&p.status->pad[0], n_pre);
    if (n_chd) atomicAdd(&p.status->pad[1], n_chd);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

size_t pre_smem_bytes(int D, int M0, int C, int Mtot) {
    const int kvs = D == 64 ? 2 : 1;
    const size_t M0p = (size_t)((M0 + 15) & ~15);
    return 1024 + 2 * kvs * (size_t)(D / 64) * kRegion + (size_t)(D / 64) * M0p * 128 +
           (((size_t)M0 * C * D * 2 + 15) & ~size_t(15)) + 128 * 4 /*sCn*/ +
           256 * 4 * 4 /*sKn, sBest, sSecond, sIdx*/ + (size_t)(C + 1) * 128 * 4 + 256 * 4 /*sPar, sLeaf*/ +
           8 * 4 + (size_t)Mtot * 4 + 8 + 7 * 8 + 16;
}

template <int D, int C>
cudaError_t launch_pre_tc(const avq_shape& s, const void* K, const void* V, const void* cb, int32_t* assign,
                          int32_t* counts, float* vsum, StatusBlock* status, cudaStream_t st) {
    const int BH = s.B * s.H;
    const int Mtot = s.M0 * (1 + s.C);
    const int M0p = (s.M0 + 15) & ~15;
    CUtensorMap tk, tv, tcb;
    if (!make_tma_bf16_3d(&tk, K, D, s.N, BH, kTile) || !make_tma_bf16_3d(&tv, V, D, s.N, BH, kTile) ||
        !make_tma_bf16_3d(&tcb, cb, D, Mtot, s.H, M0p))
        return cudaErrorInvalidValue;
    TcPreParams prm;
    prm.BH = BH;
    prm.H = s.H;
    prm.N = s.N;
    prm.M0 = s.M0;
    prm.M0p = M0p;
    prm.Mtot = Mtot;
    prm.ntiles = (s.N + kTile - 1) / kTile;
    prm.total_tiles = prm.ntiles * BH;
    prm.K = static_cast<const uint16_t*>(K);
    prm.codebook = static_cast<const uint16_t*>(cb);
    prm.assign = assign;
    prm.counts = counts;
    prm.vsum = vsum;
    prm.status = status;
    const size_t smem = pre_smem_bytes(D, s.M0, C, Mtot);
    auto kern = precompute_tc_kernel<D, C, D == 64 ? 2 : 1>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(prm.total_tiles, sms);
    kern<<<grid, kThreads, smem, st>>>(tk, tv, tcb, prm);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

bool precompute_tc_supported(const avq_shape& s) {
    if (s.dtype != AVQ_BF16 || (s.d != 64 && s.d != 128)) return false;
    if (!(s.C == 1 || s.C == 2 || s.C == 4 || s.C == 8 || s.C == 16)) return false;
    return pre_smem_bytes(s.d, s.M0, s.C, s.M0 * (1 + s.C)) <= 227 * 1024;
}

cudaError_t launch_precompute_tc(const avq_shape& s, const void* K, const void* V, const void* cb,
                                 int32_t* assign, int32_t* counts, float* vsum, StatusBlock* status,
                                 cudaStream_t st) {
#define AVQ_PRE_CASE(DD, CC) \
    if (s.d == DD && s.C == CC) return launch_pre_tc<DD, CC>(s, K, V, cb, assign, counts, vsum, status, st);
    AVQ_PRE_CASE(64, 1) AVQ_PRE_CASE(64, 2) AVQ_PRE_CASE(64, 4) AVQ_PRE_CASE(64, 8) AVQ_PRE_CASE(64, 16)
    AVQ_PRE_CASE(128, 1) AVQ_PRE_CASE(128, 2) AVQ_PRE_CASE(128, 4) AVQ_PRE_CASE(128, 8) AVQ_PRE_CASE(128, 16)
#undef AVQ_PRE_CASE
    return cudaErrorInvalidValue;
}

}  // namespace avq
