// avq_attention_tc.cu -- tensor-core (tcgen05) kernel of avq_attention for
// bf16 inputs, 128-query tiles (paper §4.3; papernotes, Key Designs 3).
//
// Persistent: one CTA of 128 threads per SM walks a contiguous range of query
// tiles (head-major, so the head's parent tables are loaded once per head).
// Thread r owns query row r of the tile and TMEM lane r.
//
// Per tile:
//   1. TMA brings the Q tile (prefetched one tile ahead, two stages).
//   2. MMA1  S_p = Q C_par^T            (M=128, N=M0p, K=d)   -> TMEM
//   3. parent pass per row: m_i = max_{n_p>0} S_ip, A_ip = e^{scale(S_ip-m_i)},
//      Zbar_i = sum_p A_ip n_p (fp32); bf16(A_ip) -> TMEM (operand of MMA3);
//      importance terms A_ip n_p / Zbar_i reduced over the 128 rows by a warp
//      butterfly and a 4-way smem sum;
//   4. top-P parents by rank counting (descending w, ties to the lower index);
//   5. per chunk of <= 128 selected children: gather their codewords and bf16
//      value sums into swizzled shared memory (cp.async), MMA2 S_c = Q C_ch^T,
//      child weights DeltaA = e^{scale(S_c-m)} - A_ip (the parent-contribution
//      replacement), fp32 denominator correction, bf16(DeltaA) -> TMEM;
//   6. MMA3  Xbar = [A_par | DeltaA] x [vsum_par ; vsum_child] accumulated in
//      TMEM (A operand from TMEM, B = bf16 value sums, MN-major);
//   7. O = Xbar / Zbar -> bf16 -> swizzled smem -> TMA store.
// One common shift m_i (the largest non-empty parent logit) is used for all
// terms of a row; any shift gives the same result in exact arithmetic, and a
// child logit more than 60 above m_i is reported as AVQ_ERANGE.
#include <algorithm>

#include "avq_internal.cuh"
#include "avq_sm100.cuh"

namespace avq {
using namespace sm100;

namespace {

constexpr int kTile = 128;
constexpr uint32_t kRegion = 128 * 128;     // one 64-column block of a 128-row image
// TMEM columns
constexpr uint32_t kColSP = 0, kColSC = 128, kColWP = 256, kColWC = 320, kColO = 384;
constexpr float kRangeLog2 = 86.56170245333781f;   // 60 / ln 2

struct TcAttnParams {
    int BH, H, N, M0, M0p, C, P, Mtot, ntiles, total_tiles;
    float sl2;                         // scale * log2(e)
    const int32_t* counts;             // [BH, Mtot]
    const uint16_t* codebook;          // [H, Mtot, D] bf16
    const uint16_t* vtab;              // [BH, Mtot, D] bf16 value sums
    int32_t* selected;                 // [BH, ntiles, P]
    StatusBlock* status;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// K-major operand, k-step ks (16 elements) of a [rows x D] bf16 image.
__device__ __forceinline__ uint64_t desc_k(const uint8_t* img, int ks) {
    const uint32_t a = smem_u32(img) + (uint32_t)(ks >> 2) * kRegion + (uint32_t)(ks & 3) * 32u;
    return smem_desc_sw128(a, 16, 1024);
}
// MN-major operand (rows = K), k-step ks covers rows 16ks..16ks+15.
__device__ __forceinline__ uint64_t desc_mn(const uint8_t* img, int ks) {
    const uint32_t a = smem_u32(img) + (uint32_t)ks * 2048u;
    return smem_desc_sw128(a, kRegion, 1024);
}
// byte offset of 16-byte chunk j (0..D/8-1) of row r in a swizzled image
__device__ __forceinline__ uint32_t swz(int r, int j) {
    return (uint32_t)(j >> 3) * kRegion + (uint32_t)r * 128u + (uint32_t)(((j & 7) ^ (r & 7)) << 4);
}

// Sum of each of 64 columns over the 32 lanes of a warp (a butterfly that
// halves the number of values each step): on return lane L holds the sums of
// columns 2L and 2L+1 in v[0], v[1].
__device__ __forceinline__ void butterfly_colsum64(float (&v)[64], int lane) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const bool up = lane & 16;
        const float keep = up ? v[j + 32] : v[j], send = up ? v[j] : v[j + 32];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const bool up = lane & 8;
        const float keep = up ? v[j + 16] : v[j], send = up ? v[j] : v[j + 16];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const bool up = lane & 4;
        const float keep = up ? v[j + 8] : v[j], send = up ? v[j] : v[j + 8];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const bool up = lane & 2;
        const float keep = up ? v[j + 4] : v[j], send = up ? v[j] : v[j + 4];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const bool up = lane & 1;
        const float keep = up ? v[j + 2] : v[j], send = up ? v[j] : v[j + 2];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
}

template <int D, int C>
__global__ void __launch_bounds__(128, 1)
attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                    const __grid_constant__ CUtensorMap tmCB, const __grid_constant__ CUtensorMap tmVT,
                    const TcAttnParams p) {
    constexpr int KH = D / 64;
    constexpr uint32_t IMG = KH * kRegion;           // bytes of one [128 x D] bf16 image
    constexpr int KSTEPS = D / 16;
    constexpr int PAR_PER_CHUNK = kTile / C;         // selected parents covered by one child chunk
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align1024(smem_raw);
    uint8_t* const sQ0 = base;                      // two Q stages: sQ0, sQ0 + IMG
    uint8_t* sB1 = base + 2 * IMG;                   // parent codewords (K-major)
    uint8_t* sB3P = base + 3 * IMG;                  // parent value sums (MN-major)
    uint8_t* sB2 = base + 4 * IMG;                   // child codewords (K-major); O staging
    uint8_t* sB3C = base + 5 * IMG;                  // child value sums (MN-major)
    float* sNp = reinterpret_cast<float*>(base + 6 * IMG);   // [128] parent counts
    float* sNc = sNp + 128;                                  // [128] child counts of the chunk
    float* sPart = sNc + 128;                                // [4][128] importance partials
    float* sW = sPart + 512;                                 // [128] importance
    int* sSel = reinterpret_cast<int*>(sW + 128);            // [128] selected parents
    uint64_t* bars = reinterpret_cast<uint64_t*>(sSel + 128);   // q0, q1, mma, head
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g0 = (int)(((long long)blockIdx.x * p.total_tiles) / gridDim.x);
    const int g1 = (int)(((long long)(blockIdx.x + 1) * p.total_tiles) / gridDim.x);

    if (warp == 0) {
        tmem_alloc(sTmem, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmO);
        tma_prefetch_desc(&tmCB);
        tma_prefetch_desc(&tmVT);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);   // this warp's lane quarter

    const uint32_t idesc1 = idesc_bf16_f32(128, p.M0p, false);
    const uint32_t idesc3 = idesc_bf16_f32(128, D, true);
    uint32_t qphase0 = 0, qphase1 = 0, mphase = 0, hphase = 0;
    bool range_bad = false;
    bool failed = false;
    int cur_bh = -1;

    auto issue_q = [&](int g, int stage) {
        const int bh = g / p.ntiles, t = g % p.ntiles;
        mbar_arrive_expect_tx(&bars[stage], IMG);
#pragma unroll
        for (int kh = 0; kh < KH; ++kh) tma_load_3d(sQ0 + stage * IMG + kh * kRegion, &tmQ, &bars[stage], kh * 64, t * kTile, bh);
    };
    if (tid == 0 && g0 < g1) issue_q(g0, 0);

    for (int g = g0, it = 0; g < g1; ++g, ++it) {
        const int stage = it & 1;
        const int bh = g / p.ntiles, t = g % p.ntiles, h = bh % p.H;
        const int rows = min(kTile, p.N - t * kTile);
        const bool valid = tid < rows;

        // previous tile's O store must have read the staging buffer (sB2)
        if (tid == 0) bulk_wait_read_all();

        if (bh != cur_bh) {   // head change: parent codewords + value sums + counts
            if (tid == 0) {
                mbar_arrive_expect_tx(&bars[3], 2u * KH * (uint32_t)p.M0p * 128u);
#pragma unroll
                for (int kh = 0; kh < KH; ++kh) {
                    tma_load_3d(sB1 + kh * kRegion, &tmCB, &bars[3], kh * 64, 0, h);
                    tma_load_3d(sB3P + kh * kRegion, &tmVT, &bars[3], kh * 64, 0, bh);
                }
            }
            sNp[tid] = tid < p.M0 ? (float)__ldg(p.counts + (size_t)bh * p.Mtot + tid) : 0.f;
            const bool ok = mbar_wait(&bars[3], hphase);
            hphase ^= 1;
            if (__syncthreads_or(!ok)) { failed = true; break; }
            cur_bh = bh;
        }

        // ---- MMA1: S_p = Q C_par^T
        bool ok = true;
        if (tid == 0) {
            ok = mbar_wait(&bars[stage], stage ? qphase1 : qphase0);
            if (stage) qphase1 ^= 1; else qphase0 ^= 1;
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks)
                    mma_ss(tmem + kColSP, desc_k(sQ0 + stage * IMG, ks), desc_k(sB1, ks), idesc1, ks > 0);
                mma_commit(&bars[2]);
                if (g + 1 < g1) issue_q(g + 1, stage ^ 1);
            }
        }
        if (__syncthreads_or(!ok)) { failed = true; break; }
        ok = mbar_wait(&bars[2], mphase);
        mphase ^= 1;
        if (__syncthreads_or(!ok)) { failed = true; break; }
        tc_fence_after();

        // ---- parent pass (16 TMEM columns at a time)
        float m = -INFINITY;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t r[16];
            tmem_ld16(trow + kColSP + 16 * c, r);
            tmem_wait_ld();
            tmem_touch16(r);
#pragma unroll
            for (int k = 0; k < 16; ++k)
                m = fmaxf(m, sNp[16 * c + k] > 0.f ? __uint_as_float(r[k]) : -INFINITY);
        }
        const float mc = m * p.sl2;
        float z = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t r[16];
            tmem_ld16(trow + kColSP + 16 * c, r);
            tmem_wait_ld();
            tmem_touch16(r);
            uint32_t w[8];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float n = sNp[16 * c + k];
                const float a = n > 0.f ? ex2(fmaf(__uint_as_float(r[k]), p.sl2, -mc)) : 0.f;
                z = fmaf(a, n, z);
                r[k] = __float_as_uint(a);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) w[k] = pack_bf16x2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
            tmem_st8(trow + kColWP + 8 * c, w);      // bf16 weights: A operand of MMA3
            tmem_st16(trow + kColSP + 16 * c, r);    // fp32 A_ip kept for the child pass
        }
        tmem_wait_st();
        // importance terms A_ip n_p / Zbar_i (zero for rows past the end)
        const float rz = valid ? 1.f / z : 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float v[64];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t r[16];
                tmem_ld16(trow + kColSP + 64 * half + 16 * c, r);
                tmem_wait_ld();
                tmem_touch16(r);
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    v[16 * c + k] = __uint_as_float(r[k]) * (sNp[64 * half + 16 * c + k] * rz);
            }
            butterfly_colsum64(v, lane);
            reinterpret_cast<float2*>(sPart + warp * 128 + 64 * half)[lane] = make_float2(v[0], v[1]);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();

        // ---- importance and top-P selection
        if (tid < p.M0) sW[tid] = (sPart[tid] + sPart[128 + tid]) + (sPart[256 + tid] + sPart[384 + tid]);
        __syncthreads();
        if (tid < p.M0) {
            const float wp = sW[tid];
            int rank = 0;
            for (int q = 0; q < p.M0; ++q) {
                const float wq = sW[q];
                rank += (wq > wp) || (wq == wp && q < tid);
            }
            if (rank < p.P) {
                sSel[rank] = tid;
                p.selected[((size_t)bh * p.ntiles + t) * p.P + rank] = tid;
            }
        }
        __syncthreads();

        // ---- children, in chunks of <= 128 slots
        float den = z;
        const int PC = p.P * C;
        const int nchunks = (PC + kTile - 1) / kTile;
        for (int k = 0; k < nchunks && !failed; ++k) {
            const int s0 = k * kTile;
            const int ns = min(kTile, PC - s0);
            const int N2 = (ns + 15) & ~15;
            // gather codewords and bf16 value sums of the chunk's children
            for (int idx = tid; idx < N2 * (D / 8); idx += 128) {
                const int slot = idx / (D / 8), j = idx % (D / 8);
                const uint32_t off = swz(slot, j);
                if (slot < ns) {
                    const int sg = s0 + slot;
                    const int child = p.M0 + sSel[sg / C] * C + (sg % C);
                    cp_async_16(sB2 + off, p.codebook + ((size_t)h * p.Mtot + child) * D + j * 8);
                    cp_async_16(sB3C + off, p.vtab + ((size_t)bh * p.Mtot + child) * D + j * 8);
                } else {
                    *reinterpret_cast<uint4*>(sB2 + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(sB3C + off) = make_uint4(0, 0, 0, 0);
                }
            }
            if (tid < kTile) {
                float nc = 0.f;
                if (tid < ns) {
                    const int sg = s0 + tid;
                    nc = (float)__ldg(p.counts + (size_t)bh * p.Mtot + p.M0 + sSel[sg / C] * C + (sg % C));
                }
                sNc[tid] = nc;
            }
            cp_async_commit();
            cp_async_wait_all();
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                if (k == 0) {   // parents' contribution (weights stored by the parent pass)
                    for (int ks = 0; ks < p.M0p / 16; ++ks)
                        mma_ts(tmem + kColO, tmem + kColWP + 8 * ks, desc_mn(sB3P, ks), idesc3, ks > 0);
                }
                const uint32_t idesc2 = idesc_bf16_f32(128, N2, false);
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks)
                    mma_ss(tmem + kColSC, desc_k(sQ0 + stage * IMG, ks), desc_k(sB2, ks), idesc2, ks > 0);
                mma_commit(&bars[2]);
            }
            ok = mbar_wait(&bars[2], mphase);
            mphase ^= 1;
            if (__syncthreads_or(!ok)) { failed = true; break; }
            tc_fence_after();

            // fp32 parent weights A_ip of the chunk's parents (kept in TMEM by the parent pass)
            float ap[PAR_PER_CHUNK];
#pragma unroll
            for (int q = 0; q < PAR_PER_CHUNK; ++q) {
                const int sidx = s0 / C + q;
                const int par = sSel[min(sidx, p.P - 1)];
                uint32_t r;
                tmem_ld1(trow + kColSP + par, r);
                tmem_wait_ld();
                tmem_touch1(r);
                ap[q] = __uint_as_float(r);
            }
            // child weights DeltaA = A_ic - A_ip, denominator correction
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t r[16];
                tmem_ld16(trow + kColSC + 16 * c, r);
                tmem_wait_ld();
                tmem_touch16(r);
                uint32_t w[8];
#pragma unroll
                for (int kk = 0; kk < 16; kk += 2) {
                    float dd[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int j = 16 * c + kk + e;
                        const float nc = sNc[j];
                        const float x = fmaf(__uint_as_float(r[kk + e]), p.sl2, -mc);
                        float dA = 0.f;
                        if (nc > 0.f) {
                            range_bad |= x > kRangeLog2;
                            dA = ex2(x) - ap[j / C];
                            den = fmaf(dA, nc, den);
                        }
                        dd[e] = dA;
                    }
                    w[kk / 2] = pack_bf16x2(dd[0], dd[1]);
                }
                // 8 packed words = the 16 child weights of this group
                tmem_st8(trow + kColWC + 8 * c, w);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                for (int ks = 0; ks < N2 / 16; ++ks)
                    mma_ts(tmem + kColO, tmem + kColWC + 8 * ks, desc_mn(sB3C, ks), idesc3, 1);
                mma_commit(&bars[2]);
            }
            ok = mbar_wait(&bars[2], mphase);
            mphase ^= 1;
            if (__syncthreads_or(!ok)) { failed = true; break; }
            tc_fence_after();
        }
        if (failed) break;
        if (nchunks == 0) {   // P == 0: parents only
            if (tid == 0) {
                tc_fence_after();
                for (int ks = 0; ks < p.M0p / 16; ++ks)
                    mma_ts(tmem + kColO, tmem + kColWP + 8 * ks, desc_mn(sB3P, ks), idesc3, ks > 0);
                mma_commit(&bars[2]);
            }
            ok = mbar_wait(&bars[2], mphase);
            mphase ^= 1;
            if (__syncthreads_or(!ok)) { failed = true; break; }
            tc_fence_after();
        }

        // ---- epilogue: O = Xbar / Zbar -> bf16 -> swizzled staging -> TMA store
        const float inv = 1.f / den;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
            uint32_t r[16];
            tmem_ld16(trow + kColO + 16 * c, r);
            tmem_wait_ld();
            tmem_touch16(r);
            uint4 a, b;
            a.x = pack_bf16x2(__uint_as_float(r[0]) * inv, __uint_as_float(r[1]) * inv);
            a.y = pack_bf16x2(__uint_as_float(r[2]) * inv, __uint_as_float(r[3]) * inv);
            a.z = pack_bf16x2(__uint_as_float(r[4]) * inv, __uint_as_float(r[5]) * inv);
            a.w = pack_bf16x2(__uint_as_float(r[6]) * inv, __uint_as_float(r[7]) * inv);
            b.x = pack_bf16x2(__uint_as_float(r[8]) * inv, __uint_as_float(r[9]) * inv);
            b.y = pack_bf16x2(__uint_as_float(r[10]) * inv, __uint_as_float(r[11]) * inv);
            b.z = pack_bf16x2(__uint_as_float(r[12]) * inv, __uint_as_float(r[13]) * inv);
            b.w = pack_bf16x2(__uint_as_float(r[14]) * inv, __uint_as_float(r[15]) * inv);
            *reinterpret_cast<uint4*>(sB2 + swz(tid, 2 * c)) = a;
            *reinterpret_cast<uint4*>(sB2 + swz(tid, 2 * c + 1)) = b;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
#pragma unroll
            for (int kh = 0; kh < KH; ++kh) tma_store_3d(&tmO, sB2 + kh * kRegion, kh * 64, t * kTile, bh);
            bulk_commit();
        }
    }

    if (range_bad) atomicExch(&p.status->error, (int)AVQ_ERANGE);
    if (failed && tid == 0) {
        atomicExch(&p.status->error, (int)AVQ_ETIMEOUT);
        atomicExch(&p.status->where, (int)blockIdx.x);
    }
    if (tid == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// bf16 copy of the value sums (B operand of the value contraction).
__global__ void vsum_to_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst, size_t n4) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const float4 v = src[i];
        uint2 o;
        o.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.x)) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.y)) << 16);
        o.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.z)) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.w)) << 16);
        dst[i] = o;
    }
}

template <int D, int C>
cudaError_t launch_tc(const avq_shape& s, const void* Q, const void* cb, const int32_t* counts, int P,
                      float scale, void* O, int32_t* selected, const void* vtab, StatusBlock* status,
                      cudaStream_t st) {
    const int BH = s.B * s.H;
    const int Mtot = s.M0 * (1 + s.C);
    const int M0p = (s.M0 + 15) & ~15;
    CUtensorMap tq, to, tcb, tvt;
    if (!make_tma_bf16_3d(&tq, Q, D, s.N, BH, kTile) || !make_tma_bf16_3d(&to, O, D, s.N, BH, kTile) ||
        !make_tma_bf16_3d(&tcb, cb, D, Mtot, s.H, M0p) || !make_tma_bf16_3d(&tvt, vtab, D, Mtot, BH, M0p))
        return cudaErrorInvalidValue;
    TcAttnParams prm;
    prm.BH = BH;
    prm.H = s.H;
    prm.N = s.N;
    prm.M0 = s.M0;
    prm.M0p = M0p;
    prm.C = s.C;
    prm.P = P;
    prm.Mtot = Mtot;
    prm.ntiles = (s.N + kTile - 1) / kTile;
    prm.total_tiles = prm.ntiles * BH;
    prm.sl2 = scale * 1.4426950408889634f;
    prm.counts = counts;
    prm.codebook = static_cast<const uint16_t*>(cb);
    prm.vtab = static_cast<const uint16_t*>(vtab);
    prm.selected = selected;
    prm.status = status;
    // Every CTA allocates all 512 TMEM columns, so at most one may be resident
    // per SM: ask for more than half of the SM's shared memory.
    const size_t smem = std::max<size_t>(1024 + 6 * (size_t)(D / 64) * kRegion + 4096 + 64, 120 * 1024);
    auto kern = attention_tc_kernel<D, C>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(prm.total_tiles, sms);
    kern<<<grid, 128, smem, st>>>(tq, to, tcb, tvt, prm);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

bool attention_tc_supported(const avq_shape& s, int tile) {
    if (s.dtype != AVQ_BF16 || tile != kTile) return false;
    if (s.d != 64 && s.d != 128) return false;
    return s.C == 1 || s.C == 2 || s.C == 4 || s.C == 8 || s.C == 16;
}

size_t attention_tc_workspace(const avq_shape& s) {
    return align256((size_t)s.B * s.H * s.M0 * (1 + s.C) * s.d * 2);
}

cudaError_t launch_attention_tc(const avq_shape& s, const void* Q, const void* cb, const int32_t* counts,
                                const float* vsum, int P, float scale, void* O, int32_t* selected,
                                void* vtab, StatusBlock* status, cudaStream_t st) {
    const size_t n4 = (size_t)s.B * s.H * s.M0 * (1 + s.C) * s.d / 4;
    vsum_to_bf16_kernel<<<(unsigned)std::min<size_t>((n4 + 255) / 256, 4096), 256, 0, st>>>(
        reinterpret_cast<const float4*>(vsum), reinterpret_cast<uint2*>(vtab), n4);
    count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
#define AVQ_TC_CASE(DD, CC) \
    if (s.d == DD && s.C == CC) return launch_tc<DD, CC>(s, Q, cb, counts, P, scale, O, selected, vtab, status, st);
    AVQ_TC_CASE(64, 1) AVQ_TC_CASE(64, 2) AVQ_TC_CASE(64, 4) AVQ_TC_CASE(64, 8) AVQ_TC_CASE(64, 16)
    AVQ_TC_CASE(128, 1) AVQ_TC_CASE(128, 2) AVQ_TC_CASE(128, 4) AVQ_TC_CASE(128, 8) AVQ_TC_CASE(128, 16)
#undef AVQ_TC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace avq
