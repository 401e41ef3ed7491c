// avq_attention_tc.cu -- tensor-core (tcgen05) kernel of avq_attention for a
// flat codebook (C == 0: VQ attention over up to 512 codewords, paper §3.2),
// and the bf16 value-means table both attention kernels contract against.
#include <algorithm>

#include "avq_internal.cuh"
#include "avq_sm100.cuh"

namespace avq {
using namespace sm100;

namespace {

constexpr int kTile = 128;
constexpr uint32_t kRegion = 128 * 128;          // one 64-column block of a 128-row image

struct TcAttnParams {
    int BH, H, N, M0, M0p, C, P, Mtot, ntiles, total_tiles;
    float sl2;                                    // scale * log2(e)
    const int32_t* counts;                        // [BH, Mtot]
    const uint16_t* codebook;                     // [H, Mtot, D] bf16
    const uint16_t* means;                        // [BH, Mtot, D] bf16 value means
    int32_t* selected;                            // [BH, ntiles, P]
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

// Packed fp32 pairs (sm_100 f32x2 arithmetic): one instruction for two lanes
// of data, each element rounded as its scalar counterpart.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
// Three-input fp32 maximum (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 32 TMEM columns of this warp's lanes into v (one wait for both loads).
__device__ __forceinline__ void tmem_ld32f(uint32_t taddr, float* v) {
    tmem_ld16f(taddr, v);
    tmem_ld16f(taddr + 16, v + 16);
    tmem_wait_ld();
    tmem_touch16f(v);
    tmem_touch16f(v + 16);
}

// pair barrier: the two warps (w and w+4) that share TMEM lanes 32w..32w+31
__device__ __forceinline__ void pair_sync(int quarter) {
    asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");
}

// Flat codebook (no children, nothing selected) with up to 512 codewords:
// VQ attention over all of them (paper §3.2: softmax weights with a
// log-count bias, per-codeword value means), in one pass over the codewords.
// They stream in chunks of 128 (codewords and means of a chunk in one of two
// TMA stages, from L2); per chunk j MMA1 writes S = Q C_j^T to TMEM, each row
// takes x_p = scale*log2(e)*S_p + log2 n_p, its chunk maximum M_j (the two
// threads of a row agree on it through shared memory) and the weights
// e'_p = 2^(x_p - m) as bf16 into TMEM, and MMA3 accumulates
// Xbar += W_j x mean_j in TMEM. The shift m is the first chunk's maximum and
// moves only when a later chunk's exceeds it by more than 2^8 (then Xbar and
// Zbar are rescaled, after the previous MMA3 has completed): the weights stay
// below 2^8, exact in relative terms in bf16 and fp32, and the common shift
// cancels in O = Xbar / Zbar. CTAs of 256 threads (two per SM at d = 64, one
// at d = 128, whose O takes 128 TMEM columns); threads r and r + 128 share
// query row r, each with half of every chunk and of the output dimensions.
template <int D>
__global__ void __launch_bounds__(256, D == 64 ? 2 : 1)
flat_attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                      const __grid_constant__ CUtensorMap tmCB, const __grid_constant__ CUtensorMap tmMN,
                      const TcAttnParams p) {
    static_assert(D == 64 || D == 128, "one or two 64-column blocks per row");
    constexpr int KH = D / 64;
    constexpr uint32_t IMG = KH * kRegion;                    // bytes of one [128 x D] bf16 image
    constexpr int KSTEPS = D / 16;
    constexpr int OD = D / 2;
    constexpr uint32_t colW = 128, colO = 192;               // TMEM: S 0..127, W 128..191, O 192..192+D
    constexpr uint32_t NCOLS = D == 64 ? 256 : 512;
    constexpr float kLazy = 8.f;                              // shift moves when a maximum exceeds it by this
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align1024(smem_raw);
    uint8_t* sQ = base;                                       // Q tile
    uint8_t* sStage = base + IMG;                             // O staging
    uint8_t* sCW = base + 2 * IMG;                            // codewords of a chunk (K-major), 2 stages
    uint8_t* sMN = base + 4 * IMG;                            // their value means (MN-major), 2 stages
    const int M0c = (p.M0 + 127) & ~127;
    const int nch = M0c / 128;
    float* sLb = reinterpret_cast<float*>(base + 6 * IMG);   // [M0c] log2 n (-inf if empty or past M0)
    float* sX = sLb + M0c;                                    // [2][2][128] chunk maxima (by chunk parity)
    float* sZ = sX + 512;                                     // [2][128] Zbar halves
    uint64_t* bars = reinterpret_cast<uint64_t*>(sZ + 256);   // Q, chunk stage 0, 1, S, O
    uint64_t* barQ = bars;
    uint64_t* barC = bars + 1;
    uint64_t* barS = bars + 3;
    uint64_t* barO = bars + 4;
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 5);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int r = tid & 127, hf = tid >> 7, quarter = warp & 3;
    const int g0 = (int)(((long long)blockIdx.x * p.total_tiles) / gridDim.x);
    const int g1 = (int)(((long long)(blockIdx.x + 1) * p.total_tiles) / gridDim.x);
    if (warp == 0) {
        tmem_alloc(sTmem, NCOLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmO);
        tma_prefetch_desc(&tmCB);
        tma_prefetch_desc(&tmMN);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t idesc3 = idesc_bf16_f32(128, D, true);
    const int M0p = (p.M0 + 15) & ~15;
    const int nchunks = (g1 - g0) * nch;                     // chunks this CTA consumes, in order
    uint32_t qph = 0, sph = 0, oph = 0;
    int cu = 0;                                               // chunks consumed: stage cu & 1
    bool failed = false;
    int cur_bh = -1;

    auto issue_q = [&](int g) {
        const int bh = g / p.ntiles, t = g % p.ntiles;
        mbar_arrive_expect_tx(barQ, IMG);
#pragma unroll
        for (int kh = 0; kh < KH; ++kh) tma_load_3d(sQ + kh * kRegion, &tmQ, barQ, kh * 64, t * kTile, bh);
    };
    // chunk c of this CTA's sequence (tile g0 + c / nch, codewords 128 (c % nch) ..) into stage c & 1
    auto issue_chunk = [&](int c) {
        const int g = g0 + c / nch, j = c % nch;
        const int bh = g / p.ntiles;
        uint64_t* bar = &barC[c & 1];
        mbar_arrive_expect_tx(bar, 2 * IMG);
#pragma unroll
        for (int kh = 0; kh < KH; ++kh) {
            tma_load_3d(sCW + (c & 1) * IMG + kh * kRegion, &tmCB, bar, kh * 64, 128 * j, bh % p.H);
            tma_load_3d(sMN + (c & 1) * IMG + kh * kRegion, &tmMN, bar, kh * 64, 128 * j, bh);
        }
    };
    // (thread 0) MMA1 of chunk c (chunk j of the current tile), once its stage landed
    auto issue_s = [&](int c, int j, bool& ok) {
        ok = mbar_wait(&barC[c & 1], (uint32_t)(c >> 1) & 1u) && ok;
        if (!ok) return;
        const int nj = min(128, M0p - 128 * j);
        const uint32_t idesc1 = idesc_bf16_f32(128, nj, false);
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks)
            mma_ss(tmem, desc_k(sQ, ks), desc_k(sCW + (c & 1) * IMG, ks), idesc1, ks > 0);
        mma_commit(barS);
    };

    if (tid == 0 && g0 < g1) {
        issue_q(g0);
        issue_chunk(0);
        if (nchunks > 1) issue_chunk(1);
    }
    for (int g = g0; g < g1; ++g) {
        const int bh = g / p.ntiles, t = g % p.ntiles;
        if (tid == 0) bulk_wait_read_all();   // the previous O store has read the staging buffer
        if (bh != cur_bh) {                   // log-counts of this (b,h)
            __syncthreads();
            for (int i = tid; i < M0c; i += 256) {
                const int n = i < p.M0 ? __ldg(p.counts + (size_t)bh * p.Mtot + i) : 0;
                sLb[i] = n > 0 ? __log2f((float)n) : -INFINITY;
            }
            __syncthreads();
            cur_bh = bh;
        }
        bool ok = true;
        if (tid == 0) {
            ok = mbar_wait(barQ, qph);
            if (ok) issue_s(cu, 0, ok);
        }
        qph ^= 1u;
        float m = -INFINITY;
        float2 z0 = make_float2(0.f, 0.f), z1 = make_float2(0.f, 0.f);
        for (int j = 0; j < nch; ++j, ++cu) {
            const int s = cu & 1;
            ok = mbar_wait(barS, sph) && ok;   // MMA1 of this chunk, and every MMA before it
            sph ^= 1u;
            tc_fence_after();
            if (tid == 0) {
                // the previous chunk's stage is free (its MMA3 preceded this MMA1)
                if (cu >= 1 && cu + 1 < nchunks) issue_chunk(cu + 1);
                if (j == nch - 1 && g + 1 < g1) issue_q(g + 1);   // the last MMA1 has read Q
            }
            // this half's 64 logits x_p in log2 units with the log-count bias:
            // first their maximum, then (below) the weights from a second read
            // of S, so that only 16 of them are live at a time
            float mx = -INFINITY;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int col = 128 * j + 64 * hf + 16 * b;
                if (col < M0p) {
                    float x[16];
                    tmem_ld16f(trow + 64 * hf + 16 * b, x);
                    tmem_wait_ld();
                    tmem_touch16f(x);
#pragma unroll
                    for (int k = 0; k < 16; k += 4) {
                        const float4 lb = *reinterpret_cast<const float4*>(sLb + col + k);
                        mx = fmax3(mx, fmaf(x[k], p.sl2, lb.x), fmaf(x[k + 1], p.sl2, lb.y));
                        mx = fmax3(mx, fmaf(x[k + 2], p.sl2, lb.z), fmaf(x[k + 3], p.sl2, lb.w));
                    }
                }
            }
            float* sXj = sX + (j & 1) * 256;
            sXj[hf * 128 + r] = mx;
            pair_sync(quarter);
            const float M = fmaxf(sXj[r], sXj[128 + r]);
            // the shift moves for a row whose maximum exceeds it by more than
            // kLazy: its Zbar and Xbar are rescaled (the MMA3s so far have
            // completed). The TMEM accesses are warp-collective, so a warp takes
            // them when any of its rows moves, with factor 1 for the others.
            const bool mv = j > 0 && M > m + kLazy;
            if (j == 0) m = M;
            if (__any_sync(0xffffffffu, mv)) {
                const float f = mv ? ex2(m - M) : 1.f;
                const float2 f2 = make_float2(f, f);
                z0 = fmul2(z0, f2);
                z1 = fmul2(z1, f2);
#pragma unroll 1
                for (int c = 0; c < OD / 16; ++c) {
                    uint32_t u[16];
                    tmem_ld16(trow + colO + hf * OD + 16 * c, u);
                    tmem_wait_ld();
                    tmem_touch16(u);
#pragma unroll
                    for (int k = 0; k < 16; ++k) u[k] = __float_as_uint(__uint_as_float(u[k]) * f);
                    tmem_st16(trow + colO + hf * OD + 16 * c, u);
                }
                if (mv) m = M;
            }
            const float2 sl2v = make_float2(p.sl2, p.sl2);
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int col = 128 * j + 64 * hf + 16 * b;
                if (col >= M0p) break;   // (columns past the codebook are not read by MMA3)
                float x[16];
                tmem_ld16f(trow + 64 * hf + 16 * b, x);
                tmem_wait_ld();
                tmem_touch16f(x);
                uint32_t w[8];
#pragma unroll
                for (int k = 0; k < 16; k += 2) {
                    const float2 lb = *reinterpret_cast<const float2*>(sLb + col + k);
                    const float2 tt = ffma2(make_float2(x[k], x[k + 1]), sl2v, fadd2(lb, make_float2(-m, -m)));
                    const float2 e = make_float2(ex2(tt.x), ex2(tt.y));
                    if ((k >> 1) & 1) z1 = fadd2(z1, e);
                    else z0 = fadd2(z0, e);
                    w[k >> 1] = pack_bf16x2(e.x, e.y);
                }
                tmem_st8(trow + colW + 32 * hf + 8 * b, w);
            }
            tmem_wait_st();
            tc_fence_before();
            if (__syncthreads_or(!ok)) { failed = true; break; }
            if (tid == 0) {   // MMA3 of this chunk, then the next chunk's MMA1
                const int nj = min(128, M0p - 128 * j);
                tc_fence_after();
                for (int ks = 0; ks < nj / 16; ++ks)
                    mma_ts(tmem + colO, tmem + colW + 8 * ks, desc_mn(sMN + s * IMG, ks), idesc3, j > 0 || ks > 0);
                if (j + 1 < nch) issue_s(cu + 1, j + 1, ok);
                else mma_commit(barO);
            }
        }
        if (failed) break;
        ok = mbar_wait(barO, oph) && ok;   // the last MMA3
        oph ^= 1u;
        tc_fence_after();
        // epilogue: O = Xbar / Zbar -> bf16 -> swizzled staging -> TMA store
        sZ[hf * 128 + r] = (z0.x + z0.y) + (z1.x + z1.y);
        pair_sync(quarter);
        const float inv = 1.f / (sZ[r] + sZ[128 + r]);
        const float2 inv2 = make_float2(inv, inv);
#pragma unroll
        for (int c = 0; c < OD / 32; ++c) {
            float o[32];
            tmem_ld32f(trow + colO + hf * OD + 32 * c, o);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t uu[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 v = fmul2(make_float2(o[8 * q + 2 * i], o[8 * q + 2 * i + 1]), inv2);
                    uu[i] = pack_bf16x2(v.x, v.y);
                }
                *reinterpret_cast<uint4*>(sStage + swz(r, hf * (OD / 8) + 4 * c + q)) =
                    make_uint4(uu[0], uu[1], uu[2], uu[3]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok)) { failed = true; break; }
        if (tid == 0) {
#pragma unroll
            for (int kh = 0; kh < KH; ++kh) tma_store_3d(&tmO, sStage + kh * kRegion, kh * 64, t * kTile, bh);
            bulk_commit();
        }
    }
    if (failed && tid == 0) {
        atomicExch(&p.status->error, (int)AVQ_ETIMEOUT);
        atomicExch(&p.status->where, (int)blockIdx.x);
    }
    if (tid == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, NCOLS);
    }
}

// bf16 value means vsum / n (0 for empty codewords): B operand of the value contraction.
__global__ void means_bf16_kernel(const float4* __restrict__ vsum, const int32_t* __restrict__ counts,
                                  uint2* __restrict__ dst, size_t nrows, int d4) {
    const size_t n4 = nrows * (size_t)d4;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const int n = __ldg(counts + i / d4);
        const float inv = n > 0 ? 1.f / (float)n : 0.f;
        const float4 v = vsum[i];
        uint2 o;
        o.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.x * inv)) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.y * inv)) << 16);
        o.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.z * inv)) |
              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.w * inv)) << 16);
        dst[i] = o;
    }
}

}  // namespace

size_t flat_attn_smem(int D, int M0) {
    const size_t M0c = (size_t)((M0 + 127) & ~127);
    return 1024 + 6 * (size_t)(D / 64) * kRegion + M0c * 4 + 768 * 4 + 5 * 8 + 16;
}

bool flat_attention_supported(const avq_shape& s, int P, int tile) {
    return s.dtype == AVQ_BF16 && (s.d == 64 || s.d == 128) && s.C == 0 && P == 0 && tile == kTile &&
           s.M0 <= 512 && flat_attn_smem(s.d, s.M0) <= 227 * 1024;
}

namespace {
template <int D>
cudaError_t launch_flat(const avq_shape& s, const void* Q, const void* cb, const int32_t* counts, const float* vsum,
                        float scale, void* O, void* means, StatusBlock* status, cudaStream_t st) {
    const size_t nrows = (size_t)s.B * s.H * s.M0;
    means_bf16_kernel<<<(unsigned)std::min<size_t>((nrows * (D / 4) + 255) / 256, 4096), 256, 0, st>>>(
        reinterpret_cast<const float4*>(vsum), counts, reinterpret_cast<uint2*>(means), nrows, D / 4);
    count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int BH = s.B * s.H;
    CUtensorMap tq, to, tcb, tmn;
    if (!make_tma_bf16_3d(&tq, Q, D, s.N, BH, kTile) || !make_tma_bf16_3d(&to, O, D, s.N, BH, kTile) ||
        !make_tma_bf16_3d(&tcb, cb, D, s.M0, s.H, 128) || !make_tma_bf16_3d(&tmn, means, D, s.M0, BH, 128))
        return cudaErrorInvalidValue;
    TcAttnParams prm{};
    prm.BH = BH;
    prm.H = s.H;
    prm.N = s.N;
    prm.M0 = s.M0;
    prm.M0p = (s.M0 + 15) & ~15;
    prm.C = 0;
    prm.P = 0;
    prm.Mtot = s.M0;
    prm.ntiles = (s.N + kTile - 1) / kTile;
    prm.total_tiles = prm.ntiles * BH;
    prm.sl2 = scale * 1.4426950408889634f;
    prm.counts = counts;
    prm.codebook = static_cast<const uint16_t*>(cb);
    prm.means = static_cast<const uint16_t*>(means);
    prm.selected = nullptr;
    prm.status = status;
    const size_t smem = flat_attn_smem(D, s.M0);
    auto kern = flat_attention_kernel<D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    kern<<<std::min(prm.total_tiles, (D == 64 ? 2 : 1) * sms), 256, smem, st>>>(tq, to, tcb, tmn, prm);
    count_launch();
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_flat_attention(const avq_shape& s, const void* Q, const void* cb, const int32_t* counts,
                                  const float* vsum, float scale, void* O, void* means, StatusBlock* status,
                                  cudaStream_t st) {
    return s.d == 64 ? launch_flat<64>(s, Q, cb, counts, vsum, scale, O, means, status, st)
                     : launch_flat<128>(s, Q, cb, counts, vsum, scale, O, means, status, st);
}

cudaError_t launch_means_bf16(const float* vsum, const int32_t* counts, void* means, size_t nrows, int d,
                              cudaStream_t st) {
    const int d4 = d / 4;
    means_bf16_kernel<<<(unsigned)std::min<size_t>((nrows * d4 + 255) / 256, 4096), 256, 0, st>>>(
        reinterpret_cast<const float4*>(vsum), counts, reinterpret_cast<uint2*>(means), nrows, d4);
    count_launch();
    return cudaGetLastError();
}

}  // namespace avq
