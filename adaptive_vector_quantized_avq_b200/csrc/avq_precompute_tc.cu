// avq_precompute_tc.cu -- tensor-core (tcgen05) kernel of avq_precompute for
// bf16 inputs (paper §4.2; papernotes, Key Designs 2; paper Table 1 rows
// "VQ assignment" and "Value aggregation").
//
// Persistent: one CTA per SM walks a contiguous range of 128-key tiles
// (head-major). The CTA runs independent 128-thread warpgroups (four at d=64,
// two at d=128), one thread per key; warpgroup w takes tiles w, w+NWG, ... of
// each (b,h) segment of the range, with its own K stage, TMEM accumulator and
// mbarriers. The CTA meets only where the (b,h) changes.
//
// Per head (when the range enters it): TMA brings the parent codewords (the B
// operand), cp.async brings the C*M0 child codewords into a shared-memory
// image whose 16-byte chunks are permuted by the parent index (so that keys
// of different parents read different banks), and all codeword norms are
// computed in fp64 and rounded once. Counts accumulate in shared memory and
// are flushed with one global atomic per non-empty codeword.
//
// Per tile and warpgroup:
//   1. TMA brings the K tile; MMA S = K C_par^T (M=128, N=M0p, K=d) into the
//      warpgroup's TMEM columns.
//   2. a1: v_p = ||C_p||^2 - 2 S_p (the expanded distance minus ||k||^2) in
//      fp32: the minimum, then the parents within the error bound of this
//      expanded form; a single one is certainly the nearest.
//   3. a2: the kept parent and its C children, v = ||C||^2 - 2 k.C with the
//      dot product on CUDA cores (bf16 x bf16 mixed-precision fma, no
//      unpacking) under a tighter bound; a child wins only when strictly
//      closer (parent first, lowest child index among equals).
//   4. a3: assign written; the key counts at its leaf (shared memory,
//      warp-aggregated) and its V row (read from global memory, coalesced) is
//      added to the leaf's value sum with 16-byte fp32 vector reductions.
// A key whose parent or leaf the bounds leave open keeps a provisional leaf
// and is listed; after its last tile the CTA decides its listed keys with
// exact fp64 distances summed in index order and moves their contributions
// where the decision changes. A second kernel then adds each parent's
// children into the parent's totals, so that a parent holds its whole
// cluster.
#include <algorithm>

#include "avq_internal.cuh"
#include "avq_sm100.cuh"

namespace avq {
using namespace sm100;

namespace {

constexpr int kTile = 128;
constexpr uint32_t kRegion = 128 * 128;

struct TcPreParams {
    int BH, H, N, M0, M0p, Mtot, ntiles, total_tiles;
    const uint16_t* K;          // [BH, N, D] bf16
    const uint16_t* V;          // [BH, N, D] bf16
    const uint16_t* codebook;   // [H, Mtot, D] bf16
    int32_t* assign;            // [BH, N]
    int32_t* counts;            // [BH, Mtot]
    float* vsum;                // [BH, Mtot, D]
    StatusBlock* status;
    long long* fix_list;        // keys (b,h,n flattened) whose decision the fp32 bounds left open,
                                // plus (nearest parent + 1) << 40 where only the leaf is open;
                                // the CTA with tiles [g0, g1) owns entries [128 g0, 128 g1)
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

__device__ __forceinline__ void red_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// Barrier over the 128 threads of one warpgroup (ids 1, 2; 0 is __syncthreads);
// the _or form also returns whether any of them passed `pred`.
__device__ __forceinline__ void wg_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }
__device__ __forceinline__ bool wg_sync_or(int id, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id)
        : "memory");
    return r != 0;
}

// acc + x*x for the bf16 x in the low / high half of w, rounded once (sm_100
// mixed-precision fma; x*x is exact in fp32, so this equals fmaf on the
// widened value)
__device__ __forceinline__ float sqacc_lo(uint32_t w, float acc) {
    float r;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tfma.rn.f32.bf16 %0, l, l, %2;\n\t}" : "=f"(r) : "r"(w), "f"(acc));
    return r;
}
__device__ __forceinline__ float sqacc_hi(uint32_t w, float acc) {
    float r;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tfma.rn.f32.bf16 %0, h, h, %2;\n\t}" : "=f"(r) : "r"(w), "f"(acc));
    return r;
}

// acc + x*c for the bf16 values in the low / high halves of kw and cw (the
// product is exact in fp32; one rounding: sm_100 mixed-precision fma).
__device__ __forceinline__ float dotacc_lo(uint32_t kw, uint32_t cw, float acc) {
    float r;
    asm("{\n\t.reg .b16 kl, kh, cl, ch;\n\tmov.b32 {kl, kh}, %1;\n\tmov.b32 {cl, ch}, %2;\n\t"
        "fma.rn.f32.bf16 %0, kl, cl, %3;\n\t}" : "=f"(r) : "r"(kw), "r"(cw), "f"(acc));
    return r;
}
__device__ __forceinline__ float dotacc_hi(uint32_t kw, uint32_t cw, float acc) {
    float r;
    asm("{\n\t.reg .b16 kl, kh, cl, ch;\n\tmov.b32 {kl, kh}, %1;\n\tmov.b32 {cl, ch}, %2;\n\t"
        "fma.rn.f32.bf16 %0, kh, ch, %3;\n\t}" : "=f"(r) : "r"(kw), "r"(cw), "f"(acc));
    return r;
}
// k . c for the key's packed bf16 row kw and a bf16 row in shared memory whose
// 16-byte chunk j lives at chunk_off(j): sixteen accumulators of d/16 terms
// each, combined pairwise, so the sum carries at most d/16 + 3 roundings.
template <int D, typename F>
__device__ __forceinline__ float dot_bf16(const uint4 (&kw)[D / 8], const uint8_t* row_base, F chunk_off) {
    float a[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = 0.f;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const uint4 w = *reinterpret_cast<const uint4*>(row_base + chunk_off(j));
        const int o = 8 * (j & 1);
        a[o + 0] = dotacc_lo(kw[j].x, w.x, a[o + 0]); a[o + 1] = dotacc_hi(kw[j].x, w.x, a[o + 1]);
        a[o + 2] = dotacc_lo(kw[j].y, w.y, a[o + 2]); a[o + 3] = dotacc_hi(kw[j].y, w.y, a[o + 3]);
        a[o + 4] = dotacc_lo(kw[j].z, w.z, a[o + 4]); a[o + 5] = dotacc_hi(kw[j].z, w.z, a[o + 5]);
        a[o + 6] = dotacc_lo(kw[j].w, w.w, a[o + 6]); a[o + 7] = dotacc_hi(kw[j].w, w.w, a[o + 7]);
    }
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) a[i] = __fadd_rn(a[i], a[i + w]);
    return a[0];
}
// ||row||^2 of a bf16 row in shared memory, summed in fp64 and rounded once
// to fp32 (error <= 2^-24 relative, to within fp64 rounding).
template <int D, typename F>
__device__ __forceinline__ float norm2_f64(const uint8_t* row_base, F chunk_off) {
    double s = 0.0;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const uint4 w = *reinterpret_cast<const uint4*>(row_base + chunk_off(j));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const double lo = (double)bf_lo(ww[e]), hi = (double)bf_hi(ww[e]);
            s = __fma_rn(lo, lo, s);
            s = __fma_rn(hi, hi, s);
        }
    }
    return __double2float_rn(s);
}

// Exact fp64 squared distance between the key (its bf16 row in registers,
// eight values per 16-byte word) and a bf16 row in global memory (read as
// 16-byte words), terms (x_j - c_j)^2 in index order with no fused operations:
// the same double as a plain sequential fp64 loop over the row.
template <int D>
__device__ __forceinline__ double exact_dist_rows(const uint4 (&kw)[D / 8], const uint16_t* c) {
    uint4 cw[D / 8];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) cw[j] = __ldg(reinterpret_cast<const uint4*>(c) + j);
    double s = 0.0;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const uint32_t xs[4] = {kw[j].x, kw[j].y, kw[j].z, kw[j].w}, cs[4] = {cw[j].x, cw[j].y, cw[j].z, cw[j].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double xv = (double)((e & 1) ? bf_hi(xs[e >> 1]) : bf_lo(xs[e >> 1]));
            const double cv = (double)((e & 1) ? bf_hi(cs[e >> 1]) : bf_lo(cs[e >> 1]));
            const double t = __dsub_rn(xv, cv);
            s = __dadd_rn(s, __dmul_rn(t, t));
        }
    }
    return s;
}

// (distance, index) minimum over a warp, the lower index among equal distances.
__device__ __forceinline__ void warp_argmin(double& d, int& i) {
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        const double od = __shfl_xor_sync(0xffffffffu, d, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (od < d || (od == d && oi < i)) { d = od; i = oi; }
    }
}

// The exact decision for one listed key (called by a whole warp): the nearest
// parent (lanes over the parents) unless the entry carries it, then the leaf
// from the parent's and its children's distances (one lane each), all fp64
// summed in index order, with the tie rules of the main loop. Where the
// provisional leaf differs, the key's count and V row move from it to the
// exact leaf. Not inlined: the main loop keeps its registers.
template <int D, int C>
__device__ __noinline__ void fix_key(long long entry, const uint16_t* K, const uint16_t* V, const uint16_t* codebook,
                                     int32_t* assign, int32_t* counts, float* vsum, int N, int H, int M0, int Mtot) {
    const int lane = threadIdx.x & 31;
    const long long key = entry & ((1LL << 40) - 1);
    int bp = (int)(entry >> 40) - 1;   // -1: the parent is open too
    const long long bh = key / N;
    const int h = (int)(bh % H);
    uint4 kw[D / 8];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) kw[j] = __ldg(reinterpret_cast<const uint4*>(K + key * D) + j);
    const uint16_t* cbh = codebook + (size_t)h * Mtot * D;
    if (bp < 0) {
        double dp = INFINITY;
        int ip = M0;
        for (int pp = lane; pp < M0; pp += 32) {
            const double d = exact_dist_rows<D>(kw, cbh + (size_t)pp * D);
            if (d < dp) { dp = d; ip = pp; }
        }
        warp_argmin(dp, ip);
        bp = ip < M0 ? ip : 0;   // (ip == M0 only for non-finite inputs)
    }
    // lanes 0..C-1: the children; lane C: the parent
    double d = INFINITY;
    if (lane <= C) d = exact_dist_rows<D>(kw, cbh + (size_t)(lane < C ? M0 + bp * C + lane : bp) * D);
    const double dpar = __shfl_sync(0xffffffffu, d, C);
    int cc = lane < C ? lane : C;
    if (lane >= C) d = INFINITY;
    warp_argmin(d, cc);
    const int leaf = d < dpar ? M0 + bp * C + cc : bp;
    const int old = assign[key];
    if (old != leaf) {
        const size_t base = (size_t)bh * Mtot;
        if (lane == 0) {
            assign[key] = leaf;
            atomicSub(counts + base + old, 1);
            atomicAdd(counts + base + leaf, 1);
        }
        for (int j = lane; j < D; j += 32) {
            const float v = __uint_as_float((uint32_t)__ldg(V + key * D + j) << 16);
            atomicAdd(vsum + (base + old) * D + j, -v);
            atomicAdd(vsum + (base + leaf) * D + j, v);
        }
    }
}

// Three-input fp32 minimum (sm_100).
__device__ __forceinline__ float fmin3(float a, float b, float c) {
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// NWG independent 128-thread pipelines (warpgroups) per CTA, one thread per
// key. Each warpgroup has its own K stage, TMEM accumulator and mbarriers
// and meets its own threads once per tile; the warpgroups share the per-head
// parent image, children image, norms and counts, and meet CTA-wide only
// where the (batch, head) changes.
template <int D, int C, int NWG>
__global__ void __launch_bounds__(128 * NWG, 1)
precompute_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmCB,
                     const TcPreParams p) {
    constexpr int KH = D / 64;
    constexpr uint32_t IMG = KH * kRegion;
    constexpr int KSTEPS = D / 16;
    constexpr int NT = 128 * NWG;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align1024p(smem_raw);
    uint8_t* sK0 = base;                           // K stage of warpgroup w: sK0 + w*IMG
    uint8_t* sB1 = base + NWG * IMG;               // parent codewords (K-major, TMA), M0p rows
    const uint32_t b1_region = (uint32_t)p.M0p * 128u;   // bytes between its 64-column blocks
    uint8_t* sCh = sB1 + KH * b1_region;           // children image [M0*C rows x D] bf16
    const size_t ch_bytes = (size_t)p.M0 * C * D * 2;
    float* sCn = reinterpret_cast<float*>(sCh + ((ch_bytes + 15) & ~size_t(15)));   // [128] parent norms
    float* sRed = sCn + 128;                       // [16]
    float* sCcn = sRed + 16;                       // [M0*C] child norms
    int* sCnt = reinterpret_cast<int*>(sCcn + p.M0 * C);   // [Mtot]
    int* sFix = sCnt + p.Mtot;                             // [1] entries this CTA listed
    uint64_t* bars = reinterpret_cast<uint64_t*>(
        (reinterpret_cast<uintptr_t>(sFix + 1) + 7) & ~uintptr_t(7));
    // bars: per warpgroup w: 2w = K stage, 2w+1 = MMA; 2*NWG = head
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 2 * NWG + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = tid >> 7, lt = tid & 127;        // warpgroup, key row within the tile
    const int wgbar = 1 + wg;
    uint64_t* barK = &bars[2 * wg];
    uint64_t* barM = &bars[2 * wg + 1];
    uint64_t* barH = &bars[2 * NWG];
    uint8_t* sK = sK0 + wg * IMG;
    const int g0 = (int)(((long long)blockIdx.x * p.total_tiles) / gridDim.x);
    const int g1 = (int)(((long long)(blockIdx.x + 1) * p.total_tiles) / gridDim.x);

    if (warp == 0) {
        tmem_alloc(sTmem, 128 * NWG);
        tmem_relinquish();
    }
    if (tid == 0) {
        *sFix = 0;
        for (int i = 0; i < 2 * NWG + 1; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmCB);
    }
    for (int i = tid; i < p.Mtot; i += NT) sCnt[i] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t trow = tmem + 128 * wg + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t idesc = idesc_bf16_f32(128, p.M0p, false);
    // expanded-form bound factor: 2 * (5d + 8) * 2^-24 (per distance, times
    // ||k||^2 + max ||C_p||^2)
    const float c_exp = 2.f * (5.f * D + 8.f) * 5.9604644775390625e-08f;

    uint32_t kph = 0, mph = 0, hph = 0;
    bool failed = false;
    int cur_bh = -1;
    float cnmax = 0.f;
    int n_pre = 0, n_chd = 0;   // fp64 re-decisions (diagnostics)

    auto issue_k = [&](int g) {   // lt == 0 of this warpgroup
        const int bh = g / p.ntiles, t = g % p.ntiles;
        mbar_arrive_expect_tx(barK, IMG);
#pragma unroll
        for (int kh = 0; kh < KH; ++kh) tma_load_3d(sK + kh * kRegion, &tmK, barK, kh * 64, t * kTile, bh);
    };
    auto flush_counts = [&](int bh) {
        for (int i = tid; i < p.Mtot; i += NT) {
            const int c = sCnt[i];
            if (c) {
                atomicAdd(p.counts + (size_t)bh * p.Mtot + i, c);
                sCnt[i] = 0;
            }
        }
    };

    for (int gs = g0; gs < g1 && !failed;) {
        // segment [gs, ge): the tiles of one (b,h) in this CTA's range
        const int bh = gs / p.ntiles, h = bh % p.H;
        const int ge = min(g1, (bh + 1) * p.ntiles);
        __syncthreads();   // every warpgroup is done with the previous segment
        // this warpgroup's first K tile of the segment (its stage is free; the
        // load overlaps the head data below)
        if (lt == 0 && gs + wg < ge) issue_k(gs + wg);
        if (cur_bh >= 0) flush_counts(cur_bh);
        bool ok = true;
        if (cur_bh < 0 || h != cur_bh % p.H) {
            if (tid == 0) {
                mbar_arrive_expect_tx(barH, KH * (uint32_t)p.M0p * 128u);
#pragma unroll
                for (int kh = 0; kh < KH; ++kh) tma_load_3d(sB1 + kh * b1_region, &tmCB, barH, kh * 64, 0, h);
            }
            const uint16_t* chg = p.codebook + ((size_t)h * p.Mtot + p.M0) * D;
            for (int idx = tid; idx < p.M0 * C * (D / 8); idx += NT) {
                const int i = idx / (D / 8), j = idx % (D / 8);
                cp_async_16(sCh + ch_off<D>(i, i / C, j), chg + (size_t)i * D + j * 8);
            }
            cp_async_commit();
            ok = mbar_wait(barH, hph);
            hph ^= 1;
            // codeword norms ||C||^2 (fp64, rounded once); +inf for padding
            // parents (p >= M0): they never win. The bounds below use the
            // largest norm of the head's parents and children.
            cp_async_wait_all();
            __syncthreads();   // the children image is complete
            float mx = 0.f;
            if (tid < 128) {
                float cn = INFINITY;
                if (tid < p.M0 && ok) {
                    cn = norm2_f64<D>(sB1, [&](int j) { return swz_off(tid, j, b1_region); });
                    mx = cn;
                }
                sCn[tid] = cn;
            }
            for (int i = tid; i < p.M0 * C; i += NT) {
                const float cn = norm2_f64<D>(sCh, [&](int j) { return ch_off<D>(i, i / C, j); });
                sCcn[i] = cn;
                mx = fmaxf(mx, cn);
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) sRed[warp] = mx;
        }
        if (__syncthreads_or(!ok)) { failed = true; break; }
        cnmax = sRed[0];
#pragma unroll
        for (int w = 1; w < NT / 32; ++w) cnmax = fmaxf(cnmax, sRed[w]);
        cur_bh = bh;

        // this warpgroup's tiles of the segment
        for (int g = gs + wg; g < ge; g += NWG) {
            const int t = g % p.ntiles;
            const int rows = min(kTile, p.N - t * kTile);
            const bool valid = lt < rows;

            // MMA: S = K C_par^T into this warpgroup's TMEM buffer
            ok = true;
            if (lt == 0) {
                ok = mbar_wait(barK, kph);
                if (ok) {
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks)
                        mma_ss(tmem + 128 * wg, desc_k128(sK, ks), desc_k128(sB1, ks, b1_region), idesc, ks > 0);
                    mma_commit(barM);
                }
            }
            kph ^= 1;
            // (if thread lt 0 could not issue the MMA, every thread's wait below times out)
            ok = mbar_wait(barM, mph) && ok;
            mph ^= 1;
            tc_fence_after();

            // this key's V row is read after the children: start bringing it to L2 now
            if (valid) {
                const char* vrow = reinterpret_cast<const char*>(p.V + ((size_t)bh * p.N + (size_t)t * kTile + lt) * D);
#pragma unroll
                for (int o = 0; o < D * 2; o += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(vrow + o));
            }

            // ---- a1: v_p = ||C_p||^2 - 2 S_p in one pass over TMEM, keeping the
            // smallest (and its index) and the second smallest (two trackers, even
            // and odd columns, merged after). A parent is certainly the nearest
            // when the runner-up lies above the error band of the smallest.
            float m1a = INFINITY, m2a = INFINITY, m1b = INFINITY, m2b = INFINITY;
            int i1a = 0, i1b = 0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                if (16 * c < p.M0p) {
                    float v16[16];
                    tmem_ld16f(trow + 16 * c, v16);
                    tmem_wait_ld();
                    tmem_touch16f(v16);
#pragma unroll
                    for (int q = 0; q < 16; q += 4) {
                        const float4 cn4 = *reinterpret_cast<const float4*>(sCn + 16 * c + q);
                        const float cnq[4] = {cn4.x, cn4.y, cn4.z, cn4.w};
#pragma unroll
                        for (int u = 0; u < 4; u += 2) {
                            const float va = fmaf(-2.f, v16[q + u], cnq[u]);
                            const float vb = fmaf(-2.f, v16[q + u + 1], cnq[u + 1]);
                            const bool la = va < m1a, lb = vb < m1b;
                            m2a = la ? m1a : fminf(m2a, va);
                            m2b = lb ? m1b : fminf(m2b, vb);
                            i1a = la ? 16 * c + q + u : i1a;
                            i1b = lb ? 16 * c + q + u + 1 : i1b;
                            m1a = la ? va : m1a;
                            m1b = lb ? vb : m1b;
                        }
                    }
                }
            }
            const bool use_a = m1a < m1b || (m1a == m1b && i1a < i1b);
            const float m = use_a ? m1a : m1b;
            const int im = use_a ? i1a : i1b;
            const float m2 = fminf(fminf(m2a, m2b), use_a ? m1b : m1a);

            // ||k||^2 straight from the bf16 key row (the row itself is
            // loaded again once the parent is known, to keep registers free)
            float kn;
            {
                float kn0 = 0.f, kn1 = 0.f;
#pragma unroll
                for (int j = 0; j < D / 8; ++j) {
                    const uint4 w = *reinterpret_cast<const uint4*>(sK + swz_off(lt, j));
                    kn0 = sqacc_lo(w.x, kn0); kn1 = sqacc_hi(w.x, kn1);
                    kn0 = sqacc_lo(w.y, kn0); kn1 = sqacc_hi(w.y, kn1);
                    kn0 = sqacc_lo(w.z, kn0); kn1 = sqacc_hi(w.z, kn1);
                    kn0 = sqacc_lo(w.w, kn0); kn1 = sqacc_hi(w.w, kn1);
                }
                kn = __fadd_rn(kn0, kn1);
            }

            // the parents within the error band of the smallest: a single one (the
            // runner-up above the band) is certainly the nearest; otherwise the key
            // is listed for the fp64 decision (parent 0 stands in until then)
            const float E = c_exp * (kn + cnmax);
            const float thr = __fadd_ru(m, 2.f * E);
            const bool single = m2 > thr;
            int bp = single ? im : 0;
            bool listed = valid && !single;
            n_pre += listed;
            // key row (packed bf16) -> registers
            uint4 kw[D / 8];
#pragma unroll
            for (int j = 0; j < D / 8; ++j) kw[j] = *reinterpret_cast<const uint4*>(sK + swz_off(lt, j));
            // the next K tile is written into this stage by TMA (the async proxy)
            // once the warpgroup meets below; the proxy fence orders these
            // shared-memory reads, not yet consumed, before that write (a barrier
            // alone orders them only against other threads' generic accesses)
            fence_proxy_async_smem();
            tc_fence_before();   // this tile's TMEM reads before the next MMA into the buffer
            if (wg_sync_or(wgbar, !ok)) { failed = true; break; }   // also: the K stage is free
            if (lt == 0 && g + NWG < ge) issue_k(g + NWG);

            // ---- a2: the kept parent and its children, v = ||C||^2 - 2 k.C with
            // the dot product on CUDA cores (bf16 x bf16 products exact, d/16 + 3
            // roundings) and fp64-rounded norms: |error| <= (d/16 + 5.5) u
            // (||k||^2 + max ||C||^2), bounded here by Ec. A child wins only when
            // strictly closer (parent first, lowest child index among equals);
            // the winner is certain when the runner-up lies more than 2 Ec above
            // it, else the key is listed for the fp64 decision.
            int leaf = bp;
            {
                const float Ec = (0.0625f * D + 7.f) * 1.0625f * 5.9604644775390625e-08f * (kn + cnmax);
                float lo = fmaf(-2.f, dot_bf16<D>(kw, sB1, [&](int j) { return swz_off(bp, j, b1_region); }),
                                sCn[bp]);
                float sec = INFINITY;
                int lo_i = -1;
#pragma unroll
                for (int c = 0; c < C; ++c) {
                    const int i = bp * C + c;
                    const float vc =
                        fmaf(-2.f, dot_bf16<D>(kw, sCh, [&](int j) { return ch_off<D>(i, bp, j); }), sCcn[i]);
                    if (vc < lo) { sec = lo; lo = vc; lo_i = c; }
                    else sec = fminf(sec, vc);
                }
                leaf = lo_i < 0 ? bp : p.M0 + bp * C + lo_i;
                const bool open = valid && !(sec - lo > 2.f * Ec);
                n_chd += open;
                listed = listed || open;
            }
            if (listed) {
                const int slot = atomicAdd(sFix, 1);
                const long long kidx = (long long)bh * p.N + (long long)t * kTile + lt;
                p.fix_list[(size_t)g0 * kTile + slot] = single ? kidx | ((long long)(bp + 1) << 40) : kidx;
            }

            // ---- a3: outputs. Counts and value sums go to the leaf only (the
            // parent itself or the child); the parents' totals are completed
            // by adding their children's when all tiles are done.
            const int kl = valid ? leaf : -1;
            if (valid) p.assign[(size_t)bh * p.N + t * kTile + lt] = leaf;
            {
                const unsigned same = __match_any_sync(0xffffffffu, kl);
                if (valid && lane == __ffs(same) - 1) atomicAdd(&sCnt[leaf], __popc(same));
            }
            // value sums: two keys of this warp per step (one per half-warp),
            // the V row read straight from global memory (coalesced), 16-byte
            // fp32 vector reductions
            {
                const int hl = lane & 15, sub = lane >> 4;
                constexpr int DPL = D / 16;   // dimensions per lane
                const size_t row0 = (size_t)bh * p.N + (size_t)t * kTile + 32 * (warp & 3);
                const uint16_t* vsrc = p.V + row0 * D + hl * DPL;
                float* vs_lane = p.vsum + (size_t)bh * p.Mtot * D + hl * DPL;
                if (D == 64) {
                    uint2 w[16];
                    int lf[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        lf[q] = __shfl_sync(0xffffffffu, kl, 2 * q + sub);
                        w[q] = make_uint2(0u, 0u);
                        if (lf[q] >= 0) w[q] = __ldg(reinterpret_cast<const uint2*>(vsrc + (size_t)(2 * q + sub) * D));
                    }
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        if (lf[q] >= 0)
                            red_v4(vs_lane + (size_t)lf[q] * D, bf_lo(w[q].x), bf_hi(w[q].x), bf_lo(w[q].y),
                                   bf_hi(w[q].y));
                } else {
                    uint4 w[16];
                    int lf[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        lf[q] = __shfl_sync(0xffffffffu, kl, 2 * q + sub);
                        w[q] = make_uint4(0u, 0u, 0u, 0u);
                        if (lf[q] >= 0) w[q] = __ldg(reinterpret_cast<const uint4*>(vsrc + (size_t)(2 * q + sub) * D));
                    }
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        if (lf[q] >= 0) {
                            float* dst = vs_lane + (size_t)lf[q] * D;
                            red_v4(dst, bf_lo(w[q].x), bf_hi(w[q].x), bf_lo(w[q].y), bf_hi(w[q].y));
                            red_v4(dst + 4, bf_lo(w[q].z), bf_hi(w[q].z), bf_lo(w[q].w), bf_hi(w[q].w));
                        }
                    }
                }
            }
        }
        if (__syncthreads_or(failed)) { failed = true; break; }
        gs = ge;
    }

    __syncthreads();
    if (!failed && cur_bh >= 0) flush_counts(cur_bh);
    // the exact decisions for the keys this CTA listed (one warp per key;
    // counts and sums are moved with global atomics, after the flush)
    if (!failed) {
        const int nf = *sFix;
        for (int e = warp; e < nf; e += NT / 32)
            fix_key<D, C>(p.fix_list[(size_t)g0 * kTile + e], p.K, p.V, p.codebook, p.assign, p.counts, p.vsum, p.N,
                          p.H, p.M0, p.Mtot);
    }
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
        tmem_dealloc(tmem, 128 * NWG);
    }
}

// Completes the parents' totals: counts[p] and vsum[p] (which so far hold the
// keys that stayed at the parent) plus those of the parent's C children. One
// warp per (b, h, parent).
template <int D, int C>
__global__ void __launch_bounds__(256) precompute_parent_totals_kernel(int BHM0, int M0, int Mtot, int32_t* counts,
                                                                       float* vsum) {
    const int w = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (w >= BHM0) return;
    const int bh = w / M0, pp = w % M0;
    const size_t prow = (size_t)bh * Mtot + pp;
    const size_t crow = (size_t)bh * Mtot + M0 + (size_t)pp * C;
    constexpr int DL = D / 32;   // dimensions per lane (2 or 4)
    float acc[DL];
#pragma unroll
    for (int e = 0; e < DL; ++e) acc[e] = vsum[prow * D + lane * DL + e];
    int cnt = 0;
#pragma unroll
    for (int c = 0; c < C; ++c) {
#pragma unroll
        for (int e = 0; e < DL; ++e) acc[e] += vsum[(crow + c) * D + lane * DL + e];
        cnt += counts[crow + c];
    }
#pragma unroll
    for (int e = 0; e < DL; ++e) vsum[prow * D + lane * DL + e] = acc[e];
    if (lane == 0) counts[prow] += cnt;
}

// Flat codebook (no children; the codebook is the M0 parents alone) with up
// to 512 codewords: nearest codeword, counts and value sums (paper §3.2, VQ
// attention without the tree). The warpgroup pipeline of the tree kernel;
// the dot products with the codewords come through the warpgroup's 128 TMEM
// columns in chunks of at most 128 codewords, twice per tile (the minimum,
// then the codewords within the error bound of it), and a key whose nearest
// codeword the bound leaves open is listed for the exact decision.
template <int D, int NWG>
__global__ void __launch_bounds__(128 * NWG, 1)
flat_precompute_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmCB,
                       const TcPreParams p) {
    constexpr int KH = D / 64;
    constexpr uint32_t IMG = KH * kRegion;
    constexpr int KSTEPS = D / 16;
    constexpr int NT = 128 * NWG;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align1024p(smem_raw);
    const int M0c = (p.M0 + 127) & ~127;                    // codeword rows held (whole 128-row boxes)
    const int nchunks = M0c / 128;
    uint8_t* sK0 = base;                                     // K stage of warpgroup w: sK0 + w*IMG
    uint8_t* sB1 = base + NWG * IMG;                         // codewords (K-major, TMA), M0c rows
    const uint32_t b1_region = (uint32_t)M0c * 128u;         // bytes between its 64-column blocks
    float* sCn = reinterpret_cast<float*>(sB1 + KH * b1_region);   // [M0c] norms (+inf past M0)
    float* sRed = sCn + M0c;                                 // [16]
    int* sCnt = reinterpret_cast<int*>(sRed + 16);           // [M0]
    int* sFix = sCnt + p.M0;                                 // [1]
    uint64_t* bars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(sFix + 1) + 7) & ~uintptr_t(7));
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 2 * NWG + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = tid >> 7, lt = tid & 127;
    const int wgbar = 1 + wg;
    uint64_t* barK = &bars[2 * wg];
    uint64_t* barM = &bars[2 * wg + 1];
    uint64_t* barH = &bars[2 * NWG];
    uint8_t* sK = sK0 + wg * IMG;
    const int g0 = (int)(((long long)blockIdx.x * p.total_tiles) / gridDim.x);
    const int g1 = (int)(((long long)(blockIdx.x + 1) * p.total_tiles) / gridDim.x);

    if (warp == 0) {
        tmem_alloc(sTmem, 128 * NWG);
        tmem_relinquish();
    }
    if (tid == 0) {
        *sFix = 0;
        for (int i = 0; i < 2 * NWG + 1; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmCB);
    }
    for (int i = tid; i < p.M0; i += NT) sCnt[i] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t trow = tmem + 128 * wg + ((uint32_t)((warp & 3) * 32) << 16);
    const float c_exp = 2.f * (5.f * D + 8.f) * 5.9604644775390625e-08f;

    uint32_t kph = 0, mph = 0, hph = 0;
    bool failed = false;
    int cur_bh = -1;
    float cnmax = 0.f;

    auto issue_k = [&](int g) {
        const int bh = g / p.ntiles, t = g % p.ntiles;
        mbar_arrive_expect_tx(barK, IMG);
#pragma unroll
        for (int kh = 0; kh < KH; ++kh) tma_load_3d(sK + kh * kRegion, &tmK, barK, kh * 64, t * kTile, bh);
    };
    auto flush_counts = [&](int bh) {
        for (int i = tid; i < p.M0; i += NT) {
            const int c = sCnt[i];
            if (c) {
                atomicAdd(p.counts + (size_t)bh * p.Mtot + i, c);
                sCnt[i] = 0;
            }
        }
    };
    // MMA of codeword chunk j into this warpgroup's TMEM columns and the wait
    // for it (thread lt 0 issues; false if a wait ran out)
    auto chunk_mma = [&](int j, bool& ok) {
        if (lt == 0 && ok) {
            const int nj = min(128, ((p.M0 + 15) & ~15) - 128 * j);
            const uint32_t idesc = idesc_bf16_f32(128, nj, false);
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks)
                mma_ss(tmem + 128 * wg, desc_k128(sK, ks), desc_k128(sB1 + j * 128 * 128, ks, b1_region), idesc,
                       ks > 0);
            mma_commit(barM);
        }
        ok = mbar_wait(barM, mph) && ok;
        mph ^= 1;
        tc_fence_after();
    };

    for (int gs = g0; gs < g1 && !failed;) {
        const int bh = gs / p.ntiles, h = bh % p.H;
        const int ge = min(g1, (bh + 1) * p.ntiles);
        __syncthreads();
        if (lt == 0 && gs + wg < ge) issue_k(gs + wg);
        if (cur_bh >= 0) flush_counts(cur_bh);
        bool ok = true;
        if (cur_bh < 0 || h != cur_bh % p.H) {
            if (tid == 0) {
                mbar_arrive_expect_tx(barH, KH * (uint32_t)M0c * 128u);
                for (int kh = 0; kh < KH; ++kh)
                    for (int r0 = 0; r0 < M0c; r0 += 128)
                        tma_load_3d(sB1 + kh * b1_region + r0 * 128, &tmCB, barH, kh * 64, r0, h);
            }
            ok = mbar_wait(barH, hph);
            hph ^= 1;
            float mx = 0.f;
            for (int i = tid; i < M0c; i += NT) {
                float cn = INFINITY;
                if (i < p.M0 && ok) {
                    cn = norm2_f64<D>(sB1, [&](int j) { return swz_off(i, j, b1_region); });
                    mx = fmaxf(mx, cn);
                }
                sCn[i] = cn;
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) sRed[warp] = mx;
        }
        if (__syncthreads_or(!ok)) { failed = true; break; }
        cnmax = sRed[0];
        for (int w = 1; w < NT / 32; ++w) cnmax = fmaxf(cnmax, sRed[w]);
        cur_bh = bh;

        for (int g = gs + wg; g < ge; g += NWG) {
            const int t = g % p.ntiles;
            const int rows = min(kTile, p.N - t * kTile);
            const bool valid = lt < rows;
            ok = true;
            if (lt == 0) ok = mbar_wait(barK, kph);
            kph ^= 1;
            // pass 1: the smallest v = ||C||^2 - 2 k.C over all chunks
            float m = INFINITY;
            for (int j = 0; j < nchunks; ++j) {
                chunk_mma(j, ok);
                for (int c = 0; c < 8; ++c) {
                    const int col = 128 * j + 16 * c;
                    if (col < ((p.M0 + 15) & ~15)) {
                        float v16[16];
                        tmem_ld16f(trow + 16 * c, v16);
                        tmem_wait_ld();
                        tmem_touch16f(v16);
#pragma unroll
                        for (int q = 0; q < 16; q += 4) {
                            const float4 cn4 = *reinterpret_cast<const float4*>(sCn + col + q);
                            m = fmin3(m, fmaf(-2.f, v16[q], cn4.x), fmaf(-2.f, v16[q + 1], cn4.y));
                            m = fmin3(m, fmaf(-2.f, v16[q + 2], cn4.z), fmaf(-2.f, v16[q + 3], cn4.w));
                        }
                    }
                }
                tc_fence_before();
                wg_sync(wgbar);   // the TMEM columns are free for the next chunk
            }
            float kn;
            {
                float kn0 = 0.f, kn1 = 0.f;
#pragma unroll
                for (int j = 0; j < D / 8; ++j) {
                    const uint4 w = *reinterpret_cast<const uint4*>(sK + swz_off(lt, j));
                    kn0 = sqacc_lo(w.x, kn0); kn1 = sqacc_hi(w.x, kn1);
                    kn0 = sqacc_lo(w.y, kn0); kn1 = sqacc_hi(w.y, kn1);
                    kn0 = sqacc_lo(w.z, kn0); kn1 = sqacc_hi(w.z, kn1);
                    kn0 = sqacc_lo(w.w, kn0); kn1 = sqacc_hi(w.w, kn1);
                }
                kn = __fadd_rn(kn0, kn1);
            }
            // pass 2: the codewords within the error band of the smallest
            // (count in the low 10 bits, their index sum above)
            const float thr = __fadd_ru(m, 2.f * c_exp * (kn + cnmax));
            int acc = 0;
            for (int j = 0; j < nchunks; ++j) {
                chunk_mma(j, ok);
                for (int c = 0; c < 8; ++c) {
                    const int col = 128 * j + 16 * c;
                    if (col < ((p.M0 + 15) & ~15)) {
                        float v16[16];
                        tmem_ld16f(trow + 16 * c, v16);
                        tmem_wait_ld();
                        tmem_touch16f(v16);
#pragma unroll
                        for (int q = 0; q < 16; ++q)
                            if (fmaf(-2.f, v16[q], sCn[col + q]) <= thr) acc += ((col + q) << 10) + 1;
                    }
                }
                tc_fence_before();
                if (j + 1 < nchunks) wg_sync(wgbar);
            }
            const bool one = (acc & 1023) == 1;
            const int bp = one ? (acc >> 10) : 0;
            const bool listed = valid && !one;
            fence_proxy_async_smem();   // the K stage's reads before its next TMA write
            if (wg_sync_or(wgbar, !ok)) { failed = true; break; }   // the K stage and TMEM are free
            if (lt == 0 && g + NWG < ge) issue_k(g + NWG);

            const int kl = valid ? bp : -1;
            if (valid) p.assign[(size_t)bh * p.N + t * kTile + lt] = bp;
            {
                const unsigned same = __match_any_sync(0xffffffffu, kl);
                if (valid && lane == __ffs(same) - 1) atomicAdd(&sCnt[bp], __popc(same));
            }
            if (listed) {
                atomicAdd(&p.status->pad[0], 1);
                const int slot = atomicAdd(sFix, 1);
                p.fix_list[(size_t)g0 * kTile + slot] = (long long)bh * p.N + (long long)t * kTile + lt;
            }
            {
                const int hl = lane & 15, sub = lane >> 4;
                constexpr int DPL = D / 16;
                const size_t row0 = (size_t)bh * p.N + (size_t)t * kTile + 32 * (warp & 3);
                const uint16_t* vsrc = p.V + row0 * D + hl * DPL;
                float* vs_lane = p.vsum + (size_t)bh * p.Mtot * D + hl * DPL;
                // all sixteen rows' loads first, then the reductions
                if (D == 64) {
                    uint2 w[16];
                    int lf[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        lf[q] = __shfl_sync(0xffffffffu, kl, 2 * q + sub);
                        w[q] = make_uint2(0u, 0u);
                        if (lf[q] >= 0) w[q] = __ldg(reinterpret_cast<const uint2*>(vsrc + (size_t)(2 * q + sub) * D));
                    }
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        if (lf[q] >= 0)
                            red_v4(vs_lane + (size_t)lf[q] * D, bf_lo(w[q].x), bf_hi(w[q].x), bf_lo(w[q].y),
                                   bf_hi(w[q].y));
                } else {
#pragma unroll
                    for (int h8 = 0; h8 < 16; h8 += 8) {   // eight rows at a time (registers)
                        uint4 w[8];
                        int lf[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            lf[q] = __shfl_sync(0xffffffffu, kl, 2 * (h8 + q) + sub);
                            w[q] = make_uint4(0u, 0u, 0u, 0u);
                            if (lf[q] >= 0)
                                w[q] = __ldg(reinterpret_cast<const uint4*>(vsrc + (size_t)(2 * (h8 + q) + sub) * D));
                        }
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            if (lf[q] >= 0) {
                                float* dst = vs_lane + (size_t)lf[q] * D;
                                red_v4(dst, bf_lo(w[q].x), bf_hi(w[q].x), bf_lo(w[q].y), bf_hi(w[q].y));
                                red_v4(dst + 4, bf_lo(w[q].z), bf_hi(w[q].z), bf_lo(w[q].w), bf_hi(w[q].w));
                            }
                        }
                    }
                }
            }
        }
        if (__syncthreads_or(failed)) { failed = true; break; }
        gs = ge;
    }

    __syncthreads();
    if (!failed && cur_bh >= 0) flush_counts(cur_bh);
    if (!failed) {
        const int nf = *sFix;
        for (int e = warp; e < nf; e += NT / 32)
            fix_key<D, 0>(p.fix_list[(size_t)g0 * kTile + e], p.K, p.V, p.codebook, p.assign, p.counts, p.vsum,
                          p.N, p.H, p.M0, p.Mtot);
    }
    if (failed && tid == 0) {
        atomicExch(&p.status->error, (int)AVQ_ETIMEOUT);
        atomicExch(&p.status->where, (int)blockIdx.x);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128 * NWG);
    }
}

size_t flat_smem_bytes(int D, int M0) {
    const int nwg = D == 64 ? 4 : 2;
    const size_t M0c = (size_t)((M0 + 127) & ~127);
    return 1024 + nwg * (size_t)(D / 64) * kRegion + (size_t)(D / 64) * M0c * 128 + M0c * 4 + 16 * 4 +
           (size_t)M0 * 4 + 4 + 8 + (2 * nwg + 1) * 8 + 16;
}

template <int D>
cudaError_t launch_flat_pre(const avq_shape& s, const void* K, const void* V, const void* cb, int32_t* assign,
                            int32_t* counts, float* vsum, StatusBlock* status, cudaStream_t st) {
    const int BH = s.B * s.H;
    CUtensorMap tk, tcb;
    if (!make_tma_bf16_3d(&tk, K, D, s.N, BH, kTile) || !make_tma_bf16_3d(&tcb, cb, D, s.M0, s.H, 128))
        return cudaErrorInvalidValue;
    TcPreParams prm;
    prm.BH = BH;
    prm.H = s.H;
    prm.N = s.N;
    prm.M0 = s.M0;
    prm.M0p = (s.M0 + 15) & ~15;
    prm.Mtot = s.M0;
    prm.ntiles = (s.N + kTile - 1) / kTile;
    prm.total_tiles = prm.ntiles * BH;
    prm.K = static_cast<const uint16_t*>(K);
    prm.V = static_cast<const uint16_t*>(V);
    prm.codebook = static_cast<const uint16_t*>(cb);
    prm.assign = assign;
    prm.counts = counts;
    prm.vsum = vsum;
    prm.status = status;
    prm.fix_list = reinterpret_cast<long long*>(reinterpret_cast<uint8_t*>(status) + kStatusBytes);
    constexpr int NWG = D == 64 ? 4 : 2;
    const size_t smem = flat_smem_bytes(D, s.M0);
    auto kern = flat_precompute_kernel<D, NWG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    kern<<<std::min(prm.total_tiles, sms), 128 * NWG, smem, st>>>(tk, tcb, prm);
    count_launch();
    return cudaGetLastError();
}

int pre_nwg(int D) { return D == 64 ? 4 : 2; }

size_t pre_smem_bytes(int D, int M0, int C, int Mtot) {
    const int nwg = pre_nwg(D);
    const size_t M0p = (size_t)((M0 + 15) & ~15);
    return 1024 + nwg * (size_t)(D / 64) * kRegion + (size_t)(D / 64) * M0p * 128 +
           (((size_t)M0 * C * D * 2 + 15) & ~size_t(15)) + 128 * 4 /*sCn*/ + 16 * 4 /*sRed*/ +
           (size_t)M0 * C * 4 /*sCcn*/ + (size_t)Mtot * 4 + 4 /*sFix*/ +
           8 + (2 * nwg + 1) * 8 + 16;
}

template <int D, int C>
cudaError_t launch_pre_tc(const avq_shape& s, const void* K, const void* V, const void* cb, int32_t* assign,
                          int32_t* counts, float* vsum, StatusBlock* status, cudaStream_t st) {
    const int BH = s.B * s.H;
    const int Mtot = s.M0 * (1 + s.C);
    const int M0p = (s.M0 + 15) & ~15;
    CUtensorMap tk, tcb;
    if (!make_tma_bf16_3d(&tk, K, D, s.N, BH, kTile) ||
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
    prm.V = static_cast<const uint16_t*>(V);
    prm.codebook = static_cast<const uint16_t*>(cb);
    prm.assign = assign;
    prm.counts = counts;
    prm.vsum = vsum;
    prm.status = status;
    // the workspace holds the status block, then the list of open keys
    prm.fix_list = reinterpret_cast<long long*>(reinterpret_cast<uint8_t*>(status) + kStatusBytes);
    const size_t smem = pre_smem_bytes(D, s.M0, C, Mtot);
    constexpr int NWG = D == 64 ? 4 : 2;
    auto kern = precompute_tc_kernel<D, C, NWG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(prm.total_tiles, sms);
    kern<<<grid, 128 * NWG, smem, st>>>(tk, tcb, prm);
    count_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int warps = BH * s.M0;
    precompute_parent_totals_kernel<D, C><<<(warps + 7) / 8, 256, 0, st>>>(warps, s.M0, Mtot, counts, vsum);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

bool flat_precompute_supported(const avq_shape& s) {
    return s.dtype == AVQ_BF16 && (s.d == 64 || s.d == 128) && s.C == 0 && s.M0 <= 512 &&
           flat_smem_bytes(s.d, s.M0) <= 227 * 1024;
}

cudaError_t launch_flat_precompute(const avq_shape& s, const void* K, const void* V, const void* cb,
                                   int32_t* assign, int32_t* counts, float* vsum, StatusBlock* status,
                                   cudaStream_t st) {
    return s.d == 64 ? launch_flat_pre<64>(s, K, V, cb, assign, counts, vsum, status, st)
                     : launch_flat_pre<128>(s, K, V, cb, assign, counts, vsum, status, st);
}

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
