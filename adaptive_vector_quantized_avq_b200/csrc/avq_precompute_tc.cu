// avq_precompute_tc.cu -- tensor-core (tcgen05) kernel of avq_precompute for
// bf16 inputs (paper §4.2; papernotes, Key Designs 2; paper Table 1 rows
// "VQ assignment" and "Value aggregation").
//
// Persistent: one 128-thread CTA per SM walks a contiguous range of 128-key
// tiles (head-major). Thread r owns key r of the tile and TMEM lane r.
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
//   3. a1: D~_p = ||k||^2 + ||C_p||^2 - 2 S_p in fp32; the smallest and the
//      runner-up. If they are not separated by the error bound of this
//      expanded form, the parents within the band are re-decided with the
//      exact fp64 distance summed in index order.
//   4. a2: the kept parent and its C children by the direct form
//      sum_j (k_j - c_j)^2 in fp32 (relative error <= (d+4)u); a candidate
//      wins only when strictly closer (parent first, lowest child index among
//      equals); the band the bound cannot separate is re-decided in fp64.
//   5. a3: assign written; counts in shared memory; the key's V row is added
//      to the parent's and (when the key moved) the child's value sum with
//      warp-wide coalesced fp32 vector reductions (one 256-byte row per
//      instruction for d = 64).
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
    const uint16_t* codebook;   // [H, Mtot, D] bf16
    int32_t* assign;            // [BH, N]
    int32_t* counts;            // [BH, Mtot]
    float* vsum;                // [BH, Mtot, D]
    StatusBlock* status;
};

__device__ __forceinline__ uint8_t* align1024p(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ uint64_t desc_k128(const uint8_t* img, int ks) {
    const uint32_t a = smem_u32(img) + (uint32_t)(ks >> 2) * kRegion + (uint32_t)(ks & 3) * 32u;
    return smem_desc_sw128(a, 16, 1024);
}
// 16-byte chunk j of row r of a TMA 128-byte-swizzled [rows x D] image
__device__ __forceinline__ uint32_t swz_off(int r, int j) {
    return (uint32_t)(j >> 3) * kRegion + (uint32_t)r * 128u + (uint32_t)(((j & 7) ^ (r & 7)) << 4);
}
// 16-byte chunk j of child row i (parent p = i / C) in the children image
template <int D>
__device__ __forceinline__ uint32_t ch_off(int i, int p, int j) {
    return (uint32_t)i * (D * 2) + (uint32_t)(((j & ~7) | ((j & 7) ^ (p & 7))) << 4);
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Squared distance of the key (fp32 registers) to a bf16 row in shared memory
// whose chunk j lives at byte offset chunk_off(j); two interleaved fp32
// accumulators, each term (k - c)^2 rounded once by the fused multiply-add.
template <int D, typename F>
__device__ __forceinline__ float direct_dist(const float (&k)[D], const uint8_t* row_base, F chunk_off) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const uint4 w = *reinterpret_cast<const uint4*>(row_base + chunk_off(j));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float t0 = __fsub_rn(k[8 * j + 2 * e], bf_lo(ww[e]));
            const float t1 = __fsub_rn(k[8 * j + 2 * e + 1], bf_hi(ww[e]));
            a0 = __fmaf_rn(t0, t0, a0);
            a1 = __fmaf_rn(t1, t1, a1);
        }
    }
    return __fadd_rn(a0, a1);
}

// Exact fp64 distance of the key (fp32 registers hold exact bf16 values) to a
// global bf16 codeword, terms in index order, no fused operations.
template <int D>
__device__ __noinline__ double exact_dist_reg(const float* k, const uint16_t* c) {
    double s = 0.0;
    for (int j = 0; j < D; ++j) {
        const double cj = (double)__uint_as_float((uint32_t)__ldg(c + j) << 16);
        const double t = __dsub_rn((double)k[j], cj);
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

template <int D, int C>
__global__ void __launch_bounds__(128, 1)
precompute_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmCB, const TcPreParams p) {
    constexpr int KH = D / 64;
    constexpr uint32_t IMG = KH * kRegion;
    constexpr int KSTEPS = D / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align1024p(smem_raw);
    uint8_t* sK0 = base;                     // K stages: sK0 + s*IMG
    uint8_t* sV0 = base + 2 * IMG;           // V stages
    uint8_t* sB1 = base + 4 * IMG;           // parent codewords (K-major, TMA)
    uint8_t* sCh = base + 5 * IMG;           // children image [M0*C rows x D] bf16
    const size_t ch_bytes = (size_t)p.M0 * C * D * 2;
    float* sCn = reinterpret_cast<float*>(sCh + ((ch_bytes + 15) & ~size_t(15)));   // [128]
    int* sCnt = reinterpret_cast<int*>(sCn + 128);                                     // [Mtot]
    int* sPar = sCnt + ((p.Mtot + 3) & ~3);                                            // [128]
    int* sLeaf = sPar + 128;                                                           // [128]
    float* sRed = reinterpret_cast<float*>(sLeaf + 128);                               // [4]
    uint64_t* bars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(sRed + 4) + 7) & ~uintptr_t(7));
    // bars: 0,1 = K stage; 2,3 = V stage; 4,5 = MMA buffer; 6 = head
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 7);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
    for (int i = tid; i < p.Mtot; i += 128) sCnt[i] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t idesc = idesc_bf16_f32(128, p.M0p, false);
    const float eps_dir = dist_eps(D);
    // expanded-form bound factor (see DESIGN notes): 2 * (5d + 8) * 2^-24
    const float c_exp = 2.f * (5.f * D + 8.f) * 5.9604644775390625e-08f;

    uint32_t kph = 0, vph = 0, mph = 0, hph = 0;   // phase bit of stage s = bit s
    bool failed = false;
    int cur_bh = -1;
    float cnmax = 0.f;
    int n_pre = 0, n_chd = 0;   // fp64 re-decisions (diagnostics)

    auto issue_kv = [&](int g, int s) {
        const int bh = g / p.ntiles, t = g % p.ntiles;
        mbar_arrive_expect_tx(&bars[s], IMG);
        mbar_arrive_expect_tx(&bars[2 + s], IMG);
#pragma unroll
        for (int kh = 0; kh < KH; ++kh) {
            tma_load_3d(sK0 + s * IMG + kh * kRegion, &tmK, &bars[s], kh * 64, t * kTile, bh);
            tma_load_3d(sV0 + s * IMG + kh * kRegion, &tmV, &bars[2 + s], kh * 64, t * kTile, bh);
        }
    };
    auto issue_mma = [&](int s) -> bool {   // tid 0 only
        const bool ok = mbar_wait(&bars[s], (kph >> s) & 1u);
        kph ^= 1u << s;
        if (!ok) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks)
            mma_ss(tmem + 128 * s, desc_k128(sK0 + s * IMG, ks), desc_k128(sB1, ks), idesc, ks > 0);
        mma_commit(&bars[4 + s]);
        return true;
    };
    auto flush_counts = [&](int bh) {
        for (int i = tid; i < p.Mtot; i += 128) {
            const int c = sCnt[i];
            if (c) {
                atomicAdd(p.counts + (size_t)bh * p.Mtot + i, c);
                sCnt[i] = 0;
            }
        }
    };

    if (tid == 0 && g0 < g1) {
        issue_kv(g0, 0);
        if (g0 + 1 < g1) issue_kv(g0 + 1, 1);
    }
    bool mma_issued_ahead = false;   // MMA of the current tile already issued

    for (int g = g0, it = 0; g < g1; ++g, ++it) {
        const int s = it & 1;
        const int bh = g / p.ntiles, t = g % p.ntiles, h = bh % p.H;
        const int rows = min(kTile, p.N - t * kTile);
        const bool valid = tid < rows;

        if (bh != cur_bh) {
            // flush the previous head's counts, load the new head's codewords
            if (cur_bh >= 0) flush_counts(cur_bh);
            if (cur_bh < 0 || h != cur_bh % p.H) {
                if (tid == 0) {
                    mbar_arrive_expect_tx(&bars[6], KH * (uint32_t)p.M0p * 128u);
#pragma unroll
                    for (int kh = 0; kh < KH; ++kh) tma_load_3d(sB1 + kh * kRegion, &tmCB, &bars[6], kh * 64, 0, h);
                }
                const uint16_t* chg = p.codebook + ((size_t)h * p.Mtot + p.M0) * D;
                for (int idx = tid; idx < p.M0 * C * (D / 8); idx += 128) {
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
                sCn[tid] = cn;
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
        if (tid == 0 && !mma_issued_ahead) ok = issue_mma(s);
        if (__syncthreads_or(!ok)) { failed = true; break; }
        ok = mbar_wait(&bars[4 + s], (mph >> s) & 1u);
        mph ^= 1u << s;
        if (__syncthreads_or(!ok)) { failed = true; break; }
        tc_fence_after();

        // key row -> fp32 registers; ||k||^2
        float k[D];
        {
            const uint8_t* kimg = sK0 + s * IMG;
#pragma unroll
            for (int j = 0; j < D / 8; ++j) {
                const uint4 w = *reinterpret_cast<const uint4*>(kimg + swz_off(tid, j));
                k[8 * j + 0] = bf_lo(w.x); k[8 * j + 1] = bf_hi(w.x);
                k[8 * j + 2] = bf_lo(w.y); k[8 * j + 3] = bf_hi(w.y);
                k[8 * j + 4] = bf_lo(w.z); k[8 * j + 5] = bf_hi(w.z);
                k[8 * j + 6] = bf_lo(w.w); k[8 * j + 7] = bf_hi(w.w);
            }
        }
        float kn = 0.f;
#pragma unroll
        for (int j = 0; j < D; ++j) kn = __fmaf_rn(k[j], k[j], kn);

        // issue the next tile's MMA into the other TMEM buffer (same head only)
        mma_issued_ahead = false;
        if (g + 1 < g1 && (g + 1) / p.ntiles == bh) {
            if (tid == 0) ok = issue_mma(s ^ 1);
            mma_issued_ahead = true;
        }

        // ---- a1: nearest parent (expanded form from the tensor-core dots)
        float best = INFINITY, second = INFINITY;
        int bp = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            if (16 * c < p.M0p) {
                uint32_t r[16];
                tmem_ld16(trow + 128 * s + 16 * c, r);
                tmem_wait_ld();
                tmem_touch16(r);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int pp = 16 * c + q;
                    float dd = fmaf(-2.f, __uint_as_float(r[q]), kn + sCn[pp]);
                    dd = pp < p.M0 ? dd : INFINITY;
                    if (dd < best) { second = best; best = dd; bp = pp; }
                    else second = fminf(second, dd);
                }
            }
        }
        const uint16_t* cbh = p.codebook + (size_t)h * p.Mtot * D;
        const float E = c_exp * (kn + cnmax);
        const bool redecide = valid && p.M0 > 1 && !(second - best > 2.f * E);
        if (__any_sync(0xffffffffu, redecide)) {
            // re-decide among the parents within the band, in fp64; the TMEM
            // reloads are warp-wide, the fp64 work only in the lanes that need it
            double eb = INFINITY;
            int ep = bp;
            for (int c = 0; c < p.M0p; c += 16) {
                uint32_t r[16];
                tmem_ld16(trow + 128 * s + c, r);
                tmem_wait_ld();
                tmem_touch16(r);
                if (redecide) {
                    for (int q = 0; q < 16; ++q) {
                        const int pp = c + q;
                        if (pp >= p.M0) break;
                        const float dd = fmaf(-2.f, __uint_as_float(r[q]), kn + sCn[pp]);
                        if (dd - best > 2.f * E) continue;
                        const double e = exact_dist_reg<D>(k, cbh + (size_t)pp * D);
                        if (e < eb) { eb = e; ep = pp; }
                    }
                }
            }
            if (redecide) {
                bp = ep;
                ++n_pre;
            }
        }

        // ---- a2: the kept parent and its children, direct form
        int leaf = bp;
        {
            const float dpar = direct_dist<D>(k, sB1 + 0, [&](int j) { return swz_off(bp, j); });
            float dch[C];
            float lo = dpar;
            int lo_i = -1;
#pragma unroll
            for (int c = 0; c < C; ++c) {
                const int i = bp * C + c;
                dch[c] = direct_dist<D>(k, sCh, [&](int j) { return ch_off<D>(i, bp, j); });
                if (dch[c] < lo) { lo = dch[c]; lo_i = c; }
            }
            bool sure = (lo_i < 0) || separated(lo, dpar, eps_dir);
#pragma unroll
            for (int c = 0; c < C; ++c)
                if (c != lo_i && !separated(lo, dch[c], eps_dir)) sure = false;
            if (sure) {
                leaf = lo_i < 0 ? bp : p.M0 + bp * C + lo_i;
            } else {
                double eb = exact_dist_reg<D>(k, cbh + (size_t)bp * D);
                int win = bp;
#pragma unroll
                for (int c = 0; c < C; ++c) {
                    if (separated(lo, dch[c], eps_dir)) continue;
                    const double e = exact_dist_reg<D>(k, cbh + (size_t)(p.M0 + bp * C + c) * D);
                    if (e < eb) { eb = e; win = p.M0 + bp * C + c; }
                }
                leaf = win;
                ++n_chd;
            }
        }

        // ---- a3: outputs
        if (tid < rows) {
            p.assign[(size_t)bh * p.N + t * kTile + tid] = leaf;
            atomicAdd(&sCnt[bp], 1);
            if (leaf != bp) atomicAdd(&sCnt[leaf], 1);
        }
        sPar[tid] = tid < rows ? bp : -1;
        sLeaf[tid] = leaf;
        if (__syncthreads_or(!ok)) { failed = true; break; }   // also: K stage s free

        // refill K stage s with tile g+2 (its V stage is refilled after the sums)
        const bool ok_v = mbar_wait(&bars[2 + s], (vph >> s) & 1u);
        vph ^= 1u << s;
        if (__syncthreads_or(!ok_v)) { failed = true; break; }

        // value sums: warp w adds the V rows of keys 32w..32w+31
        {
            const uint8_t* vimg = sV0 + s * IMG;
            float* vs_bh = p.vsum + (size_t)bh * p.Mtot * D;
            for (int q = 0; q < 32; ++q) {
                const int r = 32 * warp + q;
                const int par = sPar[r];
                if (par < 0) break;
                const int lf = sLeaf[r];
                if (D == 64) {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(vimg + swz_off(r, lane >> 2) + (lane & 3) * 4);
                    const float a = bf_lo(w), b = bf_hi(w);
                    red_v2(vs_bh + (size_t)par * D + 2 * lane, a, b);
                    if (lf != par) red_v2(vs_bh + (size_t)lf * D + 2 * lane, a, b);
                } else {
                    const uint2 w = *reinterpret_cast<const uint2*>(vimg + swz_off(r, lane >> 1) + (lane & 1) * 8);
                    const float a = bf_lo(w.x), b = bf_hi(w.x), c = bf_lo(w.y), d = bf_hi(w.y);
                    red_v4(vs_bh + (size_t)par * D + 4 * lane, a, b, c, d);
                    if (lf != par) red_v4(vs_bh + (size_t)lf * D + 4 * lane, a, b, c, d);
                }
            }
        }
        __syncthreads();
        if (tid == 0 && g + 2 < g1) issue_kv(g + 2, s);
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
    prm.codebook = static_cast<const uint16_t*>(cb);
    prm.assign = assign;
    prm.counts = counts;
    prm.vsum = vsum;
    prm.status = status;
    const size_t ch_bytes = ((size_t)s.M0 * C * D * 2 + 15) & ~size_t(15);
    const size_t smem = 1024 + 5 * (size_t)(D / 64) * kRegion + ch_bytes + 128 * 4 +
                        (((size_t)Mtot + 3) & ~size_t(3)) * 4 + 256 * 4 + 16 + 8 + 7 * 8 + 16;
    auto kern = precompute_tc_kernel<D, C>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(prm.total_tiles, sms);
    kern<<<grid, 128, smem, st>>>(tk, tv, tcb, prm);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

// Shared-memory bytes the tensor-core precompute needs (0 when it cannot run).
size_t precompute_tc_smem(const avq_shape& s) {
    const int D = s.d;
    const size_t Mtot = (size_t)s.M0 * (1 + s.C);
    return 1024 + 5 * (size_t)(D / 64) * kRegion + (((size_t)s.M0 * s.C * D * 2 + 15) & ~size_t(15)) +
           128 * 4 + ((Mtot + 3) & ~size_t(3)) * 4 + 256 * 4 + 16 + 8 + 7 * 8 + 16;
}

bool precompute_tc_supported(const avq_shape& s) {
    if (s.dtype != AVQ_BF16 || (s.d != 64 && s.d != 128)) return false;
    if (!(s.C == 1 || s.C == 2 || s.C == 4 || s.C == 8 || s.C == 16)) return false;
    return precompute_tc_smem(s) <= 227 * 1024;
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
