// avq_capture.cu -- avq_capture: top-P capture of the true attention weight
// (paper §5.2 "Elastic Inference via Top-P Adjustment", Table 6; Figure 7).
//
// For query i of head (b,h), in tile t = i / 128,
//   capture_i = sum_{k : parent(k) in sel(t)} e^{s_ik} / sum_k e^{s_ik},
//   s_ik = scale * Q_i . K_k over all N keys of the head,
// where parent(k) is the key's leaf when that is a parent (id < M0) and the
// child's parent (id - M0) / C otherwise.
//
// An exact-attention pass with no values. Persistent CTAs of 256 threads walk
// contiguous ranges of query tiles. Per query tile the key tiles of the head
// stream through shared memory (TMA, three stages); tcgen05 computes
// S = Q K^T (M = N = 128) into one of two TMEM buffers while the CUDA cores
// reduce the other into two online-softmax sums per row (all keys; keys of
// the selected parents): a per-tile fp32 partial with the running maximum as
// the shift, added to fp64 running sums that are rescaled when the maximum
// grows. Threads r and r + 128 share query row r (64 key columns each) and
// merge their sums at the end of the tile. The key masks (valid, selected
// parent) come from `assign` and the tile's selection as ballots, one word
// per 32 keys.
#include <algorithm>

#include "avq_internal.cuh"
#include "avq_sm100.cuh"

namespace avq {
using namespace sm100;

namespace {

constexpr int kT = 128;
constexpr uint32_t kBlk = 128 * 128;   // one 64-column block of a 128-row bf16 image
constexpr int kStages = 3;

struct CapParams {
    int N, M0, C, Mtot, P, ntiles, total_tiles;
    float sl2;                   // scale * log2(e)
    const int32_t* assign;       // [BH, N]
    const int32_t* selected;     // [BH, ntiles, P]
    float* capture;              // [BH, N]
    StatusBlock* status;
};

__device__ __forceinline__ uint8_t* align_1k(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
// K-major operand, k-step ks (16 elements) of a [128 x D] bf16 image.
__device__ __forceinline__ uint64_t kmajor_desc(const uint8_t* img, int ks) {
    const uint32_t a = smem_u32(img) + (uint32_t)(ks >> 2) * kBlk + (uint32_t)(ks & 3) * 32u;
    return smem_desc_sw128(a, 16, 1024);
}
// the two warps (w and w + 4) that share TMEM lanes 32w..32w+31
__device__ __forceinline__ void lane_pair_sync(int quarter) {
    asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

template <int D, int MINB>
__global__ void __launch_bounds__(256, MINB)
capture_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, const CapParams p) {
    constexpr int KH = D / 64;
    constexpr uint32_t IMG = KH * kBlk;
    constexpr int KSTEPS = D / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align_1k(smem_raw);
    uint8_t* sQ = base;
    uint8_t* sK = base + IMG;                                             // kStages key tiles
    uint32_t* sSel = reinterpret_cast<uint32_t*>(sK + kStages * IMG);     // [4] selected parents (bits)
    uint32_t* sMask = sSel + 4;                                           // [2 buffers][valid 4 | selected 4]
    float* sM = reinterpret_cast<float*>(sMask + 16);                     // [128] upper half's maximum
    double* sL = reinterpret_cast<double*>(sM + 128);                     // [2][128] upper half's sums
    uint64_t* bars = reinterpret_cast<uint64_t*>(sL + 256);               // Q, K stages, S buffers
    uint64_t* barQ = bars;
    uint64_t* barK = bars + 1;
    uint64_t* barS = bars + 1 + kStages;
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 3 + kStages);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = tid & 127, hf = tid >> 7, quarter = warp & 3;
    const int g0 = (int)(((long long)blockIdx.x * p.total_tiles) / gridDim.x);
    const int g1 = (int)(((long long)(blockIdx.x + 1) * p.total_tiles) / gridDim.x);
    const int nkt = (p.N + kT - 1) / kT;

    if (warp == 0) {
        tmem_alloc(sTmem, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 3 + kStages; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16) + 64u * hf;
    constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);

    uint32_t qph = 0;
    unsigned u = 0;      // key tiles consumed by this CTA: K stage u % kStages, S buffer u & 1
    unsigned ku = 0;     // key tiles requested (thread 0); equals u at every query-tile start
    bool failed = false;

    auto issue_k = [&](int bh, int kt) {
        const int s = (int)(ku % kStages);
        mbar_arrive_expect_tx(&barK[s], IMG);
#pragma unroll
        for (int kh = 0; kh < KH; ++kh) tma_load_3d(sK + s * IMG + kh * kBlk, &tmK, &barK[s], kh * 64, kt * kT, bh);
        ++ku;
    };
    // thread 0: S[uu & 1] = Q K^T for consumed-tile index uu, once its key tile landed
    auto issue_s = [&](unsigned uu, bool& ok) {
        const int s = (int)(uu % kStages);
        ok = mbar_wait(&barK[s], (uu / kStages) & 1u) && ok;
        if (!ok) return;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks)
            mma_ss(tmem + 128u * (uu & 1u), kmajor_desc(sQ, ks), kmajor_desc(sK + s * IMG, ks), idesc, ks > 0);
        mma_commit(&barS[uu & 1u]);
    };

    for (int g = g0; g < g1 && !failed; ++g) {
        const int bh = g / p.ntiles, t = g % p.ntiles;
        if (tid < 4) sSel[tid] = 0;
        __syncthreads();   // (every MMA and mask read of the previous tile is done)
        bool ok = true;
        if (tid == 0) {
            mbar_arrive_expect_tx(barQ, IMG);
#pragma unroll
            for (int kh = 0; kh < KH; ++kh) tma_load_3d(sQ + kh * kBlk, &tmQ, barQ, kh * 64, t * kT, bh);
            const int npre = min(kStages, nkt);
            for (int kt = 0; kt < npre; ++kt) issue_k(bh, kt);
        }
        if (tid < p.P) {
            const int v = __ldg(p.selected + (size_t)g * p.P + tid);
            if (v >= 0 && v < p.M0) atomicOr(&sSel[v >> 5], 1u << (v & 31));
        }
        const int32_t* abh = p.assign + (size_t)bh * p.N;
        int a_next = (tid < kT && tid < p.N) ? __ldg(abh + tid) : -1;
        if (tid == 0) {
            ok = mbar_wait(barQ, qph);
            issue_s(u, ok);
        }
        qph ^= 1u;
        __syncthreads();   // the selection bits

        float m = -INFINITY;          // running maximum of this thread's columns (log2 units)
        double la = 0.0, ls = 0.0;    // sums of 2^(x - m): all keys, keys of selected parents
        for (int kt = 0; kt < nkt; ++kt, ++u) {
            const unsigned buf = u & 1u;
            if (tid == 0 && kt + 1 < nkt) issue_s(u + 1, ok);
            if (tid < kT) {   // masks of this key tile
                const int a = a_next;
                const int key = kt * kT + tid;
                a_next = (key + kT < p.N) ? __ldg(abh + key + kT) : -1;
                const bool valid = key < p.N;
                int par = -1;
                if (a >= 0 && a < p.Mtot) par = a < p.M0 ? a : (a - p.M0) / p.C;
                const bool on = valid && par >= 0 && ((sSel[par >> 5] >> (par & 31)) & 1u);
                const unsigned vb = __ballot_sync(0xffffffffu, valid), sb = __ballot_sync(0xffffffffu, on);
                if (lane == 0) {
                    sMask[buf * 8 + warp] = vb;
                    sMask[buf * 8 + 4 + warp] = sb;
                }
            }
            __syncthreads();
            ok = mbar_wait(&barS[buf], (u >> 1) & 1u) && ok;
            tc_fence_after();
            float s[64];
#pragma unroll
            for (int b = 0; b < 4; ++b) tmem_ld16f(trow + 128u * buf + 16 * b, s + 16 * b);
            tmem_wait_ld();
#pragma unroll
            for (int b = 0; b < 4; ++b) tmem_touch16f(s + 16 * b);
            const uint32_t v0 = sMask[buf * 8 + 2 * hf], v1 = sMask[buf * 8 + 2 * hf + 1];
            const uint32_t w0 = sMask[buf * 8 + 4 + 2 * hf], w1 = sMask[buf * 8 + 4 + 2 * hf + 1];
            if ((v0 & v1) != 0xffffffffu) {   // past the last key (ragged last key tile)
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    if (!((v0 >> k) & 1u)) s[k] = -INFINITY;
                    if (!((v1 >> k) & 1u)) s[32 + k] = -INFINITY;
                }
            }
            float mt = s[63];
#pragma unroll
            for (int k = 0; k < 62; k += 2) mt = max3f(mt, s[k], s[k + 1]);
            mt = fmaxf(mt, s[62]) * p.sl2;
            if (mt > m) {   // the maximum grows: rescale the running sums
                const double f = (double)ex2(m - mt);   // 0 when m = -inf
                la *= f;
                ls *= f;
                m = mt;
            }
            const float nm = m == -INFINITY ? 0.f : -m;
            float pa0 = 0.f, pa1 = 0.f, ps0 = 0.f, ps1 = 0.f;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float e0 = ex2(fmaf(s[k], p.sl2, nm)), e1 = ex2(fmaf(s[32 + k], p.sl2, nm));
                pa0 += e0;
                pa1 += e1;
                ps0 += ((w0 >> k) & 1u) ? e0 : 0.f;
                ps1 += ((w1 >> k) & 1u) ? e1 : 0.f;
            }
            la += (double)(pa0 + pa1);
            ls += (double)(ps0 + ps1);
            tc_fence_before();
            if (__syncthreads_or(!ok)) { failed = true; break; }
            // key tile kt's stage is free (its MMA completed): request tile kt + kStages
            if (tid == 0 && kt + kStages < nkt) issue_k(bh, kt + kStages);
        }
        if (failed) break;
        if (hf == 1) {
            sM[r] = m;
            sL[r] = la;
            sL[128 + r] = ls;
        }
        lane_pair_sync(quarter);
        if (hf == 0) {
            const float m1 = sM[r], mm = fmaxf(m, m1);
            const double f0 = m == -INFINITY ? 0.0 : (double)ex2(m - mm);
            const double f1 = m1 == -INFINITY ? 0.0 : (double)ex2(m1 - mm);
            const double all = la * f0 + sL[r] * f1, sel = ls * f0 + sL[128 + r] * f1;
            const int row = t * kT + r;
            if (row < p.N) p.capture[(size_t)bh * p.N + row] = (float)(sel / all);
        }
        lane_pair_sync(quarter);
    }

    if (failed && tid == 0) {
        atomicExch(&p.status->error, (int)AVQ_ETIMEOUT);
        atomicExch(&p.status->where, (int)blockIdx.x);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

template <int D>
size_t capture_smem() {
    const size_t img = (size_t)(D / 64) * kBlk;
    const size_t need = 1024 + (1 + kStages) * img + 16 + 64 + 128 * 4 + 256 * 8 + (3 + kStages) * 8 + 16;
    // at d = 64 two CTAs (256 TMEM columns each) share an SM; more than 76 KB
    // keeps a third one off it
    return D == 64 ? std::max<size_t>(need, 80 * 1024) : need;
}

template <int D>
cudaError_t launch_capture(const avq_shape& s, const void* Q, const void* K, const int32_t* assign,
                           const int32_t* selected, int P, float scale, float* capture, StatusBlock* status,
                           cudaStream_t st) {
    constexpr int MINB = D == 64 ? 2 : 1;
    const int BH = s.B * s.H;
    CUtensorMap tq, tk;
    if (!make_tma_bf16_3d(&tq, Q, D, s.N, BH, kT) || !make_tma_bf16_3d(&tk, K, D, s.N, BH, kT))
        return cudaErrorInvalidValue;
    CapParams prm;
    prm.N = s.N;
    prm.M0 = s.M0;
    prm.C = s.C;
    prm.Mtot = s.M0 * (1 + s.C);
    prm.P = P;
    prm.ntiles = (s.N + kT - 1) / kT;
    prm.total_tiles = prm.ntiles * BH;
    prm.sl2 = scale * 1.4426950408889634f;
    prm.assign = assign;
    prm.selected = selected;
    prm.capture = capture;
    prm.status = status;
    const size_t smem = capture_smem<D>();
    auto kern = capture_kernel<D, MINB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    kern<<<std::min(prm.total_tiles, sms * MINB), 256, smem, st>>>(tq, tk, prm);
    count_launch();
    return cudaGetLastError();
}

bool capture_supported(const avq_shape& s, int tile) { return s.dtype == AVQ_BF16 && tile == kT; }

}  // namespace
}  // namespace avq

using namespace avq;

namespace {
int capture_args(const avq_shape* s, int P, int tile) {
    if (!s) return AVQ_EINVAL;
    if (s->B < 1 || s->H < 1 || s->N < 0 || (s->d != 64 && s->d != 128)) return AVQ_EINVAL;
    if (s->dtype != AVQ_F32 && s->dtype != AVQ_BF16) return AVQ_EINVAL;
    if (s->M0 < 1 || s->C < 0) return AVQ_EINVAL;
    if (s->M0 > (s->C == 0 ? kMaxFlat : kMaxM0) || s->C > kMaxC) return AVQ_EUNSUPPORTED;
    if ((long long)s->B * s->H * s->N * s->d >= (1LL << 40)) return AVQ_EUNSUPPORTED;
    if (P < 0 || P > s->M0 || (tile != 64 && tile != 128)) return AVQ_EINVAL;
    if (s->C == 0 && P != 0) return AVQ_EINVAL;   // a flat codebook selects nothing
    if (!capture_supported(*s, tile)) return AVQ_EUNSUPPORTED;
    return AVQ_OK;
}
}  // namespace

extern "C" size_t avq_capture_workspace_bytes(const avq_shape* s, int P, int tile) {
    return capture_args(s, P, tile) == AVQ_OK ? kStatusBytes : 0;
}

extern "C" int avq_capture(const avq_shape* s, const void* Q, const void* K, const int32_t* assign,
                           const int32_t* selected, int P, int tile, float scale, float* capture, void* workspace,
                           size_t workspace_bytes, void* stream) {
    if (!s) return AVQ_EINVAL;
    // argument errors before unsupported cases, as the other entry points
    if (s->B < 1 || s->H < 1 || s->N < 0 || (s->d != 64 && s->d != 128)) return AVQ_EINVAL;
    if (P < 0 || P > s->M0 || (tile != 64 && tile != 128)) return AVQ_EINVAL;
    if (!(scale > 0.f) || !(scale < 3.0e38f)) return AVQ_EINVAL;
    const auto al = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0; };
    if (s->N > 0 && (!capture || !Q || !K || !assign || (P > 0 && !selected))) return AVQ_EINVAL;
    if (!al(Q, 16) || !al(K, 16) || !al(assign, 4) || !al(selected, 4) || !al(capture, 4)) return AVQ_EINVAL;
    const int rc = capture_args(s, P, tile);
    if (rc != AVQ_OK) return rc;
    if (!workspace || workspace_bytes < kStatusBytes || !al(workspace, 16)) return AVQ_EWORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, kStatusBytes, st) != cudaSuccess) return AVQ_ECUDA;
    if (s->N == 0) return AVQ_OK;
    const size_t rows = (size_t)s->B * s->H * s->N;
    if (P == 0)   // nothing selected: no weight is captured
        return cudaMemsetAsync(capture, 0, rows * sizeof(float), st) == cudaSuccess ? AVQ_OK : AVQ_ECUDA;
    StatusBlock* status = static_cast<StatusBlock*>(workspace);
    const cudaError_t e = s->d == 64 ? launch_capture<64>(*s, Q, K, assign, selected, P, scale, capture, status, st)
                                     : launch_capture<128>(*s, Q, K, assign, selected, P, scale, capture, status, st);
    return e == cudaSuccess ? AVQ_OK : AVQ_ECUDA;
}
