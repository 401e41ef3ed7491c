// avq_attention_tree.cu -- tensor-core (tcgen05) kernel of avq_attention for
// bf16 trees, 128-query tiles (paper §4.3; papernotes, Key Designs 3).
//
// Persistent. A CTA has 256 threads, two per query row (warps w and w + 4
// share the TMEM lanes of the row; each takes every other 16-column block of
// the parents, of the child slots and half of the output dimensions). Thread
// 0 also issues the loads of Q and of the head's parent tables (TMA) and
// every tcgen05.mma, each right after the CTA barrier that already orders
// its inputs; mbarriers carry only the tensor core's and TMA's completions.
// The next tile's S = Q C^T is issued ahead of the current tile's last value
// contraction, and each tile's epilogue runs one tile late, under the next
// tile's first parent pass. Two CTAs share an SM at d = 64.
//
// TMEM (columns; 256 at d = 64, 512 at d = 128):
//   [0, 128)          S_p = Q C_par^T (fp32); then e'_p (fp32) for the
//                     importance; then S_c = Q C_child^T of a chunk of up to
//                     128 child slots, and that chunk's child weights W_c
//                     (bf16) over the read S_c columns
//   [128, 128 + d)    O (fp32): Xbar accumulated by the value contractions
//   [128 + d, +64)    W_p (bf16): the parents' weights (A operand); the
//                     tile's last chunk of child weights goes over it, so
//                     that the next tile's S_p can be computed while the
//                     last value contraction still reads them
//
// Weights are kept in log-count form: x_p = scale*log2(e)*S_p + log2 n_p, so
// e'_p = 2^(x_p - m) = A_p n_p with one shift m per row (the largest x_p).
// The value contractions use per-codeword value MEANS (vsum / n), so
//   Xbar = W_p x mean_par + sum_chunks W_c x mean_child,
// and the denominator Zbar is summed from exactly the bf16 weights the
// contractions multiply (each weight rounded once, then used on both
// sides). Per tile:
//   1. MMA1 S_p; parent pass: x_p, m, e'_p, Zbar (fp32, exact, for the
//      importance), bf16 W_p -> TMEM; MMA3p O = W_p x mean_par (issued once
//      every thread's W_p is written).
//   2. Importance w_p = sum_rows e'_p / Zbar, from TMEM in the 16x256b
//      layout (each thread holds four rows), a three-level butterfly and a
//      four-warp sum in shared memory; top-P over 64-bit values (the bit
//      pattern of w >= 0 above the complement of the index: ties to the lower
//      index), each of four warps sorting 32 of them, a value's rank found
//      by binary searches in the other warps' lists.
//   3. Per chunk of <= 128 selected child slots: the children's codewords and
//      value means are gathered (TMA, else cp.async), thread 0 issues MMA2
//      S_c; the child weight (A_c - A_p) n_c = 2^(x_c - m) -
//      A_p n_c (the ΔA replacement of the papernotes summary in
//      count-weighted form, A_p taken from the bf16 W_p that MMA3p used) ->
//      bf16 W_c; MMA3c.
//   4. O = Xbar / Zbar -> bf16 -> swizzled staging -> TMA store (one tile
//      late).
// A child logit far above the row's shift (more than 64 octaves) moves the
// shift: the row's O, W_p, denominator and written child weights are scaled
// by an exact power of two (paper §4.3: the running accumulators are
// rescaled whenever the maximum changes).
#include <algorithm>
#include <atomic>

#include "avq_internal.cuh"
#include "avq_sm100.cuh"

namespace avq {

// (test hook, see avq_test_fail_next_wait) the next tree attention launch gives
// up thread 0's first wait at once
std::atomic<int> g_fail_next_wait{0};

cudaError_t launch_means_bf16(const float* vsum, const int32_t* counts, void* means, size_t nrows, int d,
                              cudaStream_t st);

namespace {
using namespace sm100;

constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr int kBars = 8;                  // mbarriers in shared memory
constexpr uint32_t kRegion = 128 * 128;   // one 64-column block of a 128-row bf16 image
constexpr float kRescale = 64.f;          // largest child weight exponent (log2) before the shift moves

struct TreeParams {
    int BH, H, N, M0, M0p, C, P, Mtot, ntiles, total_tiles;
    float sl2;                   // scale * log2(e)
    uint32_t colO, colWp, ncols;
    const int32_t* counts;       // [BH, Mtot]
    const uint16_t* codebook;    // [H, Mtot, D] bf16
    const uint16_t* means;       // [BH, Mtot, D] bf16 value means
    int32_t* selected;           // [BH, ntiles, P]
    StatusBlock* status;
    int fail_first_wait;         // (test hook) thread 0's first wait gives up at once
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
// K-major operand, k-step ks (16 elements) of a [rows x D] bf16 image
__device__ __forceinline__ uint64_t desc_k(const uint8_t* img, int ks) {
    const uint32_t a = smem_u32(img) + (uint32_t)(ks >> 2) * kRegion + (uint32_t)(ks & 3) * 32u;
    return smem_desc_sw128(a, 16, 1024);
}
// MN-major operand (rows = K), k-step ks covers rows 16ks .. 16ks + 15
__device__ __forceinline__ uint64_t desc_mn(const uint8_t* img, int ks) {
    const uint32_t a = smem_u32(img) + (uint32_t)ks * 2048u;
    return smem_desc_sw128(a, kRegion, 1024);
}
// byte offset of 16-byte chunk j of row r in a swizzled image
__device__ __forceinline__ uint32_t swz(int r, int j) {
    return (uint32_t)(j >> 3) * kRegion + (uint32_t)r * 128u + (uint32_t)(((j & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
// 2^-k for an integer 0 <= k (0 below the normal range)
__device__ __forceinline__ float exp2_neg_int(int k) { return k < 127 ? __int_as_float((127 - k) << 23) : 0.f; }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// the compute threads' barrier (named barrier 1, 256 threads), OR of a flag
__device__ __forceinline__ bool wg_sync_or(bool flag) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)flag)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void wg_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// the two warps (w and w + 4) that share the TMEM lanes of quarter q
__device__ __forceinline__ void pair_sync(int q) { asm volatile("bar.sync %0, 64;" ::"r"(2 + q) : "memory"); }

// Waits for the phase with the given parity; gives up (false) when another
// thread of the CTA gave up or after one second (then it tells the others).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > 1000000000ull) {
            *abort = 1;
            return false;
        }
    }
}

// 16 lanes x 256 bits, twice (16 columns): thread t receives, per 8-column
// group g, the columns 2(t%4), 2(t%4)+1 of lanes t/4 (r[4g], r[4g+1]) and
// t/4 + 8 (r[4g+2], r[4g+3]).
__device__ __forceinline__ void tmem_ld_16x256b_x2(uint32_t taddr, float* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16f(uint32_t taddr, const float* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
        "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* u) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
                 : "r"(taddr));
}
__device__ __forceinline__ void touch8u(uint32_t* u) {
    asm volatile("" : "+r"(u[0]), "+r"(u[1]), "+r"(u[2]), "+r"(u[3]), "+r"(u[4]), "+r"(u[5]), "+r"(u[6]), "+r"(u[7]));
}
__device__ __forceinline__ void touch8f(float* v) {
    asm volatile("" : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]), "+f"(v[7]));
}

// One butterfly level over 2H values: lanes with `up` keep the upper half and
// send the lower one, the others the reverse; kept values add the partner's.
template <int H>
__device__ __forceinline__ void butterfly_level(float* v, bool up, int mask) {
#pragma unroll
    for (int j = 0; j < H; j += 2) {
        const float k0 = up ? v[j + H] : v[j], s0 = up ? v[j] : v[j + H];
        const float k1 = up ? v[j + 1 + H] : v[j + 1], s1 = up ? v[j + 1] : v[j + 1 + H];
        const float r0 = __shfl_xor_sync(0xffffffffu, s0, mask);
        const float r1 = __shfl_xor_sync(0xffffffffu, s1, mask);
        const float2 o = fadd2(make_float2(k0, k1), make_float2(r0, r1));
        v[j] = o.x;
        v[j + 1] = o.y;
    }
}

// The tile's top-P parents, in rank order, into sel (shared) and out (global),
// by four warps (quarter q holds parents 32q .. 32q + 31, one per lane). Each
// parent's value is the bit pattern of its importance w >= 0 (which orders like
// w) above the complement of its index, so that ties go to the lower index;
// parents past M0 sort last. Each warp sorts its 32 values (bitonic, 15
// shuffle steps) and publishes them; a value's rank is its place in its own
// list plus, for each other list, the number of larger values there (a binary
// search). list: 128 64-bit words of shared memory.
__device__ __forceinline__ void select_top_p4(const float* part, unsigned long long* list, int* sel, int32_t* out,
                                              int M0, int P, int q, int lane) {
    const int par = 32 * q + lane;
    const float w = (part[par] + part[128 + par]) + (part[256 + par] + part[384 + par]);
    const uint32_t key = par < M0 ? __float_as_uint(w) : 0u;
    unsigned long long v = ((unsigned long long)key << 32) | (uint32_t)(0xFFFFFFFFu - par);
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, j);
            v = (v > o) == keep_max ? v : o;
        }
    }
    list[32 * q + lane] = v;
    asm volatile("bar.sync 6, 128;" ::: "memory");
    if (lane < P) {
        int rank = lane;
#pragma unroll
        for (int d = 1; d < 4; ++d) {
            const unsigned long long* L = list + 32 * ((q + d) & 3);
            int c = 0;   // number of values in L above v (L is descending)
#pragma unroll
            for (int step = 16; step > 0; step >>= 1)
                if (L[c + step - 1] > v) c += step;
            c += L[c] > v;   // (c <= 31 here)
            rank += c;
        }
        if (rank < P) {
            const int pr = (int)(0xFFFFFFFFu - (uint32_t)v);
            sel[rank] = pr;
            out[rank] = pr;
        }
    }
}

// FULL: 128 parents, so that each thread's parent blocks number four (fixed
// loop counts)
template <int D, int C, int MINB, bool FULL>
__global__ void __launch_bounds__(kThreads, MINB)
attention_tree_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                      const __grid_constant__ CUtensorMap tmCB, const __grid_constant__ CUtensorMap tmMN,
                      const __grid_constant__ CUtensorMap tmCBc, const __grid_constant__ CUtensorMap tmMNc,
                      const TreeParams p) {
    constexpr int KH = D / 64;
    constexpr uint32_t IMG = KH * kRegion;   // bytes of one [128 x D] bf16 image
    constexpr int KSTEPS = D / 16;
    constexpr int OD = D / 2;                // output dimensions per thread of a row
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align1024(smem_raw);
    uint8_t* const sQ = base;                // two Q stages
    uint8_t* const sCP = base + 2 * IMG;     // parent codewords (K-major)
    uint8_t* const sMP = base + 3 * IMG;     // parent value means (MN-major)
    uint8_t* const sCC = base + 4 * IMG;     // child codewords of a chunk (K-major)
    uint8_t* const sMC = base + 5 * IMG;     // their value means (MN-major); O staging
    float* sLb = reinterpret_cast<float*>(base + 6 * IMG);   // [128] log2 n_p (-inf if empty)
    float* sInvN = sLb + 128;                // [128] 1 / n_p
    float* sRz = sInvN + 128;                // [128] 1 / Zbar per row (0 past the end)
    float* sPart = sRz + 128;                // [4][128] importance partials per quarter
    float* sNc = sPart + 512;                // [128] child counts of the chunk's slots
    float* sLc = sNc + 128;                  // [128] their log2 (-inf if empty)
    float* sX = sLc + 128;                   // [2][128] row exchange: shift; the selection's sorted lists
    float* sZ = sX + 256;                    // [2][128] row exchange: Zbar, then the denominator
    float* sT = sZ + 256;                    // [2][128] row exchange: largest child exponent
    int* sSel = reinterpret_cast<int*>(sT + 256);              // [128] selected parents by rank
    // [128] per selected parent: its W_p column (offset from colWp), and the
    // bits of 1 / n_p with the sign bit set when its weight is the low bf16 half
    uint2* sLk = reinterpret_cast<uint2*>(sSel + 128);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sLk + 128);
    uint64_t* bQ = bars;                     // [2] Q stage landed
    uint64_t* bHead = bars + 2;              // head tables landed
    uint64_t* bS = bars + 3;                 // MMA1 / MMA2 done (S_p, S_c ready)
    uint64_t* bO = bars + 4;                 // the tile's last contraction done
    uint64_t* bC = bars + 5;                 // a chunk's contraction done (all but the last)
    uint64_t* bFin = bars + 6;               // (failure only) contractions in flight done
    uint64_t* bGatT = bars + 7;              // (P + 1, tx) the selected parents' children landed (TMA)
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + kBars);
    volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);
    float* sCnt = reinterpret_cast<float*>(sTmem + 4);        // [M0 * C] this (b,h)'s child counts

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3;                  // TMEM lane quarter of this warp
    const int hf = warp >> 2;                // which half of the row's columns
    const int r = 32 * q + lane;             // query row (and parent / slot index)
    const bool leader = tid == 0;            // issues the Q and head loads and every tcgen05.mma
    const bool store_thread = tid == 32;     // issues the O stores
    const int g0 = (int)(((long long)blockIdx.x * p.total_tiles) / gridDim.x);
    const int g1 = (int)(((long long)(blockIdx.x + 1) * p.total_tiles) / gridDim.x);
    const int PC = p.P * C;
    const int nchunks = (PC + 127) / 128;    // chunks of up to 128 child slots
    // the children of each selected parent are C contiguous codebook (and means)
    // rows: with C a multiple of 8 they fill whole 1 KB swizzle atoms, and a
    // single chunk's gather is one TMA load per selected parent and image
    const bool tma_gather = (C % 8 == 0) && nchunks == 1;

    if (warp == 0) {
        tmem_alloc(sTmem, p.ncols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) mbar_init(&bQ[i], 1);
        mbar_init(bHead, 1);
        mbar_init(bS, 1);
        mbar_init(bO, 1);
        mbar_init(bC, 1);
        mbar_init(bFin, 1);
        mbar_init(bGatT, tma_gather ? p.P + 1 : 1);
        *sAbort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmO);
        tma_prefetch_desc(&tmCB);
        tma_prefetch_desc(&tmMN);
        tma_prefetch_desc(&tmCBc);
        tma_prefetch_desc(&tmMNc);
    }
    // child images start finite (padding slots are read by MMA2 and weighted by 0)
    for (int i = tid; i < 2 * (int)IMG / 16; i += kThreads)
        reinterpret_cast<uint4*>(sCC)[i] = make_uint4(0, 0, 0, 0);   // sCC and sMC are adjacent
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    bool failed = false;
    // (leader) loads issued but not yet seen complete, for the failure path
    uint32_t q_pending = 0, qph = 0, hph = 0, gtph = 0;
    bool head_pending = false, gat_pending = false;
    const uint32_t idesc1 = idesc_bf16_f32(128, p.M0p, false);
    const uint32_t idesc3 = idesc_bf16_f32(128, D, true);
    // (leader) the TMA load of tile g's Q into stage `stage`
    auto issue_q = [&](int g, int stage) {
        const int bh = g / p.ntiles, t = g % p.ntiles;
        q_pending |= 1u << stage;
        mbar_arrive_expect_tx(&bQ[stage], IMG);
#pragma unroll
        for (int kh = 0; kh < KH; ++kh)
            tma_load_3d(sQ + stage * IMG + kh * kRegion, &tmQ, &bQ[stage], kh * 64, t * kTile, bh);
    };
    // (leader) MMA1 S_p = Q C_par^T of tile g (its Q in stage `stage`), then the
    // load of the next tile's Q into the other stage (free: every contraction
    // that read it is complete); false when the wait for Q gave up
    auto issue_mma1 = [&](int g, int stage) -> bool {
        if (!wait_bar(&bQ[stage], (qph >> stage) & 1u, sAbort)) return false;
        qph ^= 1u << stage;
        q_pending &= ~(1u << stage);
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks)
            mma_ss(tmem, desc_k(sQ + stage * IMG, ks), desc_k(sCP, ks), idesc1, ks > 0);
        mma_commit(bS);
        if (g + 1 < g1) issue_q(g + 1, stage ^ 1);
        return true;
    };

    const int ct = tid;
    const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16);
    uint32_t sph = 0, oph = 0, cph = 0;
    int cur_bh = -1;
    bool mma1_chained = false;   // (leader) this tile's MMA1 went out at the end of the previous tile
    const float2 sl2v = make_float2(p.sl2, p.sl2);
    bool ok = true;
    // ---- epilogue of tile (et, ebh): O = Xbar / Zbar -> bf16 -> swizzled
    // staging -> TMA store (this thread: output dimensions hf * OD .. + OD - 1).
    // It runs one tile late, after the next tile's first parent pass, so that
    // the tile's last contraction completes under that pass. True when a wait
    // gave up (for every thread).
    auto epilogue = [&](int et, int ebh, float eden) -> bool {
        sZ[hf * 128 + r] = eden;
        ok = wait_bar(bO, oph, sAbort) && ok;
        oph ^= 1;
        tc_fence_after();
        uint32_t packed[OD / 2];
        {
            float o[OD];
#pragma unroll
            for (int c = 0; c < OD / 16; ++c) tmem_ld16f(trow + p.colO + hf * OD + 16 * c, o + 16 * c);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < OD / 16; ++c) tmem_touch16f(o + 16 * c);
            tc_fence_before();
            pair_sync(q);
            const float inv = 1.f / (sZ[r] + sZ[128 + r]);
            const float2 inv2 = make_float2(inv, inv);
#pragma unroll
            for (int i = 0; i < OD / 2; ++i) {
                const float2 v2 = fmul2(make_float2(o[2 * i], o[2 * i + 1]), inv2);
                packed[i] = pack_bf16x2(v2.x, v2.y);
            }
        }
        if (PC == 0 && store_thread) bulk_wait_read_all();
        if (wg_sync_or(!ok)) return true;   // (and: the staging buffer is free)
#pragma unroll
        for (int j = 0; j < OD / 8; ++j)
            *reinterpret_cast<uint4*>(sMC + swz(r, hf * (OD / 8) + j)) =
                make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
        fence_proxy_async_smem();
        wg_sync();
        if (store_thread) {
#pragma unroll
            for (int kh = 0; kh < KH; ++kh) tma_store_3d(&tmO, sMC + kh * kRegion, kh * 64, et * kTile, ebh);
            bulk_commit();
        }
        return false;
    };
    bool pend = false;   // a tile whose epilogue is still to run
    int pend_t = 0, pend_bh = 0;
    float pend_den = 0.f;
    if (leader && g0 < g1) issue_q(g0, 0);
    for (int g = g0, it = 0; g < g1; ++g, ++it) {
        const int stage = it & 1;
        const int bh = g / p.ntiles, t = g % p.ntiles, h = bh % p.H;
        // the next tile's MMA1 goes out with this tile's last contraction when it
        // uses the same parent tables
        const bool chain_next = g + 1 < g1 && (g + 1) / p.ntiles == bh;
        const int rows = min(kTile, p.N - t * kTile);
        const bool valid = r < rows;
        if (bh != cur_bh) {   // this (b,h)'s parent tables, log-counts and child counts
            if (pend) {       // the previous tile's output first (its contractions end there)
                if (epilogue(pend_t, pend_bh, pend_den)) { failed = true; break; }
                pend = false;
            }
            wg_sync();        // (every thread is past the previous tile, whose contractions are done)
            if (leader) {     // parent codewords and parent means (TMA)
                head_pending = true;
                mbar_arrive_expect_tx(bHead, 2u * KH * (uint32_t)p.M0p * 128u);
#pragma unroll
                for (int kh = 0; kh < KH; ++kh) {
                    tma_load_3d(sCP + kh * kRegion, &tmCB, bHead, kh * 64, 0, h);
                    tma_load_3d(sMP + kh * kRegion, &tmMN, bHead, kh * 64, 0, bh);
                }
            }
            __syncwarp();
            if (ct < 128) {
                const int n = ct < p.M0 ? __ldg(p.counts + (size_t)bh * p.Mtot + ct) : 0;
                sLb[ct] = n > 0 ? __log2f((float)n) : -INFINITY;
                sInvN[ct] = n > 0 ? 1.f / (float)n : 0.f;
            }
            if (PC > 0)
                for (int i = ct; i < p.M0 * C; i += 256) sCnt[i] = (float)__ldg(p.counts + (size_t)bh * p.Mtot + p.M0 + i);
            wg_sync();
            cur_bh = bh;
        }
        if (leader && !mma1_chained) {   // MMA1 S_p = Q C_par^T
            if (head_pending) {
                if (it == 0 && p.fail_first_wait) {   // (test hook) a wait whose limit is zero, and ran out
                    ok = false;
                    *sAbort = 1;
                } else {
                    ok = wait_bar(bHead, hph, sAbort);
                }
                if (ok) {
                    hph ^= 1;
                    head_pending = false;
                }
            }
            ok = ok && issue_mma1(g, stage);
        }
        __syncwarp();   // (warp 0 converged again after its leader's part)
        mma1_chained = false;
        ok = wait_bar(bS, sph, sAbort) && ok;
        sph ^= 1;
        tc_fence_after();

        // ---- parent pass over this thread's 16-column blocks 2i + hf:
        // x_p = sl2 S_p + log2 n_p, the row's shift m, e'_p = 2^(x_p - m),
        // Zbar (exact) and the denominator of the rounded weights. Two
        // passes over S_p (the shift, then the weights), one block at a time.
        float m, den;
        bool epi_failed = false;
        {
            const int nbp = FULL ? 4 : (p.M0p / 16 + 1 - hf) / 2;   // this thread's parent blocks
            float mp0 = -INFINITY, mp1 = -INFINITY;
            for (int i = 0; i < nbp; ++i) {
                const int b = 2 * i + hf;
                float x[16];
                tmem_ld16f(trow + 16 * b, x);
                tmem_wait_ld();
                tmem_touch16f(x);
#pragma unroll
                for (int k = 0; k < 16; k += 4) {
                    const float4 lb = *reinterpret_cast<const float4*>(sLb + 16 * b + k);
                    const float2 a2 = ffma2(make_float2(x[k], x[k + 1]), sl2v, make_float2(lb.x, lb.y));
                    const float2 b2 = ffma2(make_float2(x[k + 2], x[k + 3]), sl2v, make_float2(lb.z, lb.w));
                    mp0 = fmax3(mp0, a2.x, a2.y);
                    mp1 = fmax3(mp1, b2.x, b2.y);
                }
            }
            sX[hf * 128 + r] = fmaxf(mp0, mp1);
            pair_sync(q);
            m = fmaxf(sX[r], sX[128 + r]);
            if (pend) {   // the previous tile's output (its last contraction ran under the pass above)
                epi_failed = epilogue(pend_t, pend_bh, pend_den);
                pend = false;
            }
        }
        if (epi_failed) { failed = true; break; }
        {
            const int nbp = FULL ? 4 : (p.M0p / 16 + 1 - hf) / 2;
            const float2 negm = make_float2(-m, -m);
            float2 z0 = make_float2(0.f, 0.f), z1 = make_float2(0.f, 0.f);
            float2 zb0 = make_float2(0.f, 0.f), zb1 = make_float2(0.f, 0.f);
            for (int i = 0; i < nbp; ++i) {
                const int b = 2 * i + hf;
                float x[16];
                tmem_ld16f(trow + 16 * b, x);
                tmem_wait_ld();
                tmem_touch16f(x);
                uint32_t w[8];
#pragma unroll
                for (int k = 0; k < 16; k += 4) {
                    const float4 lb = *reinterpret_cast<const float4*>(sLb + 16 * b + k);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int o = k + 2 * e;
                        const float2 xx = ffma2(make_float2(x[o], x[o + 1]), sl2v,
                                                e ? make_float2(lb.z, lb.w) : make_float2(lb.x, lb.y));
                        const float2 tt = fadd2(xx, negm);
                        const float2 ev = make_float2(ex2(tt.x), ex2(tt.y));
                        x[o] = ev.x;
                        x[o + 1] = ev.y;
                        const uint32_t wb = pack_bf16x2(ev.x, ev.y);
                        const float2 er = make_float2(bf16_lo(wb), bf16_hi(wb));
                        if (e) { z1 = fadd2(z1, ev); zb1 = fadd2(zb1, er); }
                        else { z0 = fadd2(z0, ev); zb0 = fadd2(zb0, er); }
                        w[o >> 1] = wb;
                    }
                }
                tmem_st8(trow + p.colWp + 8 * b, w);
                if (PC > 0) tmem_st16f(trow + 16 * b, x);
            }
            sZ[hf * 128 + r] = (z0.x + z0.y) + (z1.x + z1.y);
            den = (zb0.x + zb0.y) + (zb1.x + zb1.y);
            pair_sync(q);
            const float z = sZ[r] + sZ[128 + r];
            sRz[r] = valid ? 1.f / z : 0.f;   // (both threads of the row write the same value)
        }
        tmem_wait_st();
        tc_fence_before();   // (the W_p writes precede MMA3p, issued after a barrier)

        if (PC > 0) {
            // ---- importance w_p = sum over the tile's rows of e'_p / Zbar
            // (each warp: its 32 rows, its four 16-column blocks)
            __syncwarp();   // this warp's rows' 1/Zbar
            {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = 0.f;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int rlo = 32 * q + 16 * hh + (lane >> 2);
                    const float2 rz = make_float2(sRz[rlo], sRz[rlo + 8]);
                    float e[32];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int b = 2 * i + hf;
                        if (FULL || 16 * b < p.M0p) {
                            tmem_ld_16x256b_x2(tmem + ((uint32_t)(32 * q + 16 * hh) << 16) + 16 * b, e + 8 * i);
                        } else {
#pragma unroll
                            for (int k = 0; k < 8; ++k) e[8 * i + k] = 0.f;
                        }
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 4; ++i) touch8f(e + 8 * i);
                    // register 4g + j of block 2i + hf: column 16(2i + hf) + 8g + 2(lane % 4) +
                    // (j % 2) of row rlo (j < 2) or rlo + 8 (j >= 2); v index 4i + 2g + (j % 2)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int gg = 0; gg < 2; ++gg) {
                            const float* ee = e + 8 * i + 4 * gg;
                            float2 acc = make_float2(v[4 * i + 2 * gg], v[4 * i + 2 * gg + 1]);
                            acc = ffma2(make_float2(ee[0], ee[1]), make_float2(rz.x, rz.x), acc);
                            acc = ffma2(make_float2(ee[2], ee[3]), make_float2(rz.y, rz.y), acc);
                            v[4 * i + 2 * gg] = acc.x;
                            v[4 * i + 2 * gg + 1] = acc.y;
                        }
                }
                // sum over the 8 lanes that hold the same columns (lane bits 2..4)
                butterfly_level<8>(v, lane & 16, 16);
                butterfly_level<4>(v, lane & 8, 8);
                butterfly_level<2>(v, lane & 4, 4);
                // v[e] = column 16(2i + hf) + 8g + 2(lane % 4) + e over the warp's rows,
                // with i = (lane >> 3) & 3... : lane bits 4, 3 give i, bit 2 gives g
                const int ii = 2 * ((lane >> 4) & 1) + ((lane >> 3) & 1), gg = (lane >> 2) & 1;
                const int c0 = 16 * (2 * ii + hf) + 8 * gg + 2 * (lane & 3);
                *reinterpret_cast<float2*>(sPart + q * 128 + c0) = make_float2(v[0], v[1]);
            }
            tc_fence_before();   // the reads of e' precede MMA2 (issued after later barriers)
            if (wg_sync_or(!ok)) { failed = true; break; }
            if (leader) {   // MMA3p O = W_p x mean_par (W_p is complete)
                tc_fence_after();
                for (int ks = 0; ks < p.M0p / 16; ++ks)
                    mma_ts(tmem + p.colO, tmem + p.colWp + 8 * ks, desc_mn(sMP, ks), idesc3, ks > 0);
            }
            __syncwarp();

            // ---- top-P: the parents ordered by (importance, then the lower
            // index), the first P selected in rank order (select_top_p4)
            if (hf == 0)
                select_top_p4(sPart, reinterpret_cast<unsigned long long*>(sX), sSel,
                              p.selected + ((size_t)bh * p.ntiles + t) * p.P, p.M0, p.P, q, lane);
            if (store_thread) bulk_wait_read_all();   // the previous O store has read the staging
            wg_sync();   // the selection is in sSel
            gat_pending = tma_gather;   // (leader: the gather below is in flight until bGatT completes)
            if (ct < p.P) {   // where the child pass finds each selected parent's weight
                const int pid = min(max(sSel[ct], 0), p.M0 - 1);
                sLk[ct] = make_uint2((uint32_t)(pid >> 1),
                                     __float_as_uint(sInvN[pid]) | ((pid & 1) ? 0u : 0x80000000u));
            }
            {
                if (tma_gather) {   // each selected parent's children: one TMA load per image
                    // (slot s from thread 32 (s % 8) + s / 8: the loads leave from all
                    // eight warps, not one warp's lanes in turn)
                    const int gslot = (ct & 31) * 8 + (ct >> 5);
                    if (gslot < p.P) {
                        const int par = min(max(sSel[gslot], 0), p.M0 - 1);
                        mbar_arrive_expect_tx(bGatT, 2u * KH * (uint32_t)C * 128u);
#pragma unroll
                        for (int kh = 0; kh < KH; ++kh) {
                            tma_load_3d(sCC + kh * kRegion + gslot * C * 128, &tmCBc, bGatT, kh * 64, p.M0 + par * C, h);
                            tma_load_3d(sMC + kh * kRegion + gslot * C * 128, &tmMNc, bGatT, kh * 64, p.M0 + par * C, bh);
                        }
                    }
                    if (ct < PC) {   // slot tables: the child's count and its log2
                        const float nc = sCnt[min(max(sSel[ct / C], 0), p.M0 - 1) * C + ct % C];
                        sNc[ct] = nc;
                        sLc[ct] = nc > 0.f ? __log2f(nc) : -INFINITY;
                    }
                }
                if (tma_gather && ct == 255) {   // the chunk's padding slots: zero rows, empty entries
                    const int N2 = (PC + 15) & ~15;
                    for (int slot = PC; slot < N2; ++slot) {
                        sNc[slot] = 0.f;
                        sLc[slot] = -INFINITY;
#pragma unroll
                        for (int j = 0; j < D / 8; ++j) {
                            *reinterpret_cast<uint4*>(sCC + swz(slot, j)) = make_uint4(0, 0, 0, 0);
                            *reinterpret_cast<uint4*>(sMC + swz(slot, j)) = make_uint4(0, 0, 0, 0);
                        }
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(bGatT);
                }
            }

            // ---- children, chunk by chunk
            for (int k = 0; k < nchunks; ++k) {
                const int cs = 128 * k;
                const int ns = min(128, PC - cs);
                const int N2 = (ns + 15) & ~15;
                if (!tma_gather) {
                if (k > 0) {
                    ok = wait_bar(bC, cph, sAbort) && ok;      // the previous chunk's MMA3c is done
                    cph ^= 1;
                }
                wg_sync();   // the selection is complete; the previous chunk's tables are no longer read
                // slot tables and the gather of the chunk's child codewords and value means
                if (ct < N2) {
                    float nc = 0.f;
                    if (ct < ns) {
                        const int sg = cs + ct;
                        nc = sCnt[min(max(sSel[sg / C], 0), p.M0 - 1) * C + (sg % C)];
                    }
                    sNc[ct] = nc;
                    sLc[ct] = nc > 0.f ? __log2f(nc) : -INFINITY;
                }
                for (int idx = ct; idx < N2 * (D / 8); idx += 256) {
                    const int slot = idx / (D / 8), j = idx % (D / 8);
                    const uint32_t off = swz(slot, j);
                    if (slot < ns) {
                        const int sg = cs + slot;
                        const int child = p.M0 + min(max(sSel[sg / C], 0), p.M0 - 1) * C + (sg % C);
                        cp_async_16(sCC + off, p.codebook + ((size_t)h * p.Mtot + child) * D + j * 8);
                        cp_async_16(sMC + off, p.means + ((size_t)bh * p.Mtot + child) * D + j * 8);
                    } else {
                        *reinterpret_cast<uint4*>(sCC + off) = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4*>(sMC + off) = make_uint4(0, 0, 0, 0);
                    }
                }
                cp_async_wait_all();
                fence_proxy_async_smem();
                wg_sync();   // the chunk's children are in shared memory
                }
                if (leader) {   // MMA2 S_c = Q C_child^T
                    if (tma_gather) {
                        ok = wait_bar(bGatT, gtph, sAbort) && ok;
                        if (ok) {
                            gtph ^= 1;
                            gat_pending = false;
                        }
                    }
                    if (ok) {
                        tc_fence_after();
                        const uint32_t idesc2 = idesc_bf16_f32(128, N2, false);
#pragma unroll
                        for (int ks = 0; ks < KSTEPS; ++ks)
                            mma_ss(tmem, desc_k(sQ + stage * IMG, ks), desc_k(sCC, ks), idesc2, ks > 0);
                        mma_commit(bS);
                    } else {
                        *sAbort = 1;   // (the others' wait for S_c gives up too)
                    }
                }
                __syncwarp();
                ok = wait_bar(bS, sph, sAbort) && ok;
                sph ^= 1;
                tc_fence_after();
                wg_sync();           // the slot tables and the selection are complete
                // child weights (A_c - A_p) n_c = 2^t - A_p n_c with t = sl2 S_c +
                // log2 n_c - m, over this thread's 16-slot blocks 2i + hf, rounded to
                // bf16 once; the denominator from the same rounded values. They are
                // held until both threads of the row have read their S_c, then
                // written as W_c over the S_c columns. When the row's largest t is
                // above 64 the shift moves up by whole octaves: O, W_p and the
                // denominator are scaled by 2^-k (exact) and the weights taken again
                // (paper §4.3: the running accumulators follow the maximum).
                const int nb = (N2 / 16 + 1 - hf) / 2;
                float2 dc0, dc1;
                uint32_t wall[4][8];
#pragma unroll 1
                for (int attempt = 0;; ++attempt) {
                    const float2 negm = make_float2(-m, -m);
                    float tmax = -INFINITY;
                    dc0 = make_float2(0.f, 0.f);
                    dc1 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (i >= nb) break;
                        const int b = 2 * i + hf;
                        constexpr int PB = C >= 16 ? 1 : 16 / C;   // parents behind a 16-slot block
                        float sc[16];
                        float nap[PB];
                        {
                            uint32_t wr[PB], code[PB];
                            tmem_ld16f(trow + 16 * b, sc);
#pragma unroll
                            for (int j = 0; j < PB; ++j) {   // -A_p = -W_p / n_p of the block's parents
                                const uint2 lk = sLk[min((cs + 16 * b) / C + j, p.P - 1)];
                                code[j] = lk.y;
                                tmem_ld1(trow + p.colWp + lk.x, wr[j]);
                            }
                            tmem_wait_ld();
                            tmem_touch16f(sc);
#pragma unroll
                            for (int j = 0; j < PB; ++j) {
                                tmem_touch1(wr[j]);
                                const uint32_t w = (wr[j] << ((code[j] >> 27) & 16u)) & 0xFFFF0000u;
                                nap[j] = __uint_as_float(code[j] | 0x80000000u) * __uint_as_float(w);
                            }
                        }
#pragma unroll
                        for (int kk = 0; kk < 16; kk += 4) {
                            const float4 lc = *reinterpret_cast<const float4*>(sLc + 16 * b + kk);
                            const float4 nc = *reinterpret_cast<const float4*>(sNc + 16 * b + kk);
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int s = kk + 2 * e;
                                const float2 tt = ffma2(make_float2(sc[s], sc[s + 1]), sl2v,
                                                        fadd2(e ? make_float2(lc.z, lc.w) : make_float2(lc.x, lc.y), negm));
                                tmax = fmax3(tmax, tt.x, tt.y);
                                const float2 ev = make_float2(ex2(tt.x), ex2(tt.y));
                                const float2 wc = ffma2(make_float2(nap[s / C < PB ? s / C : 0], nap[(s + 1) / C < PB ? (s + 1) / C : 0]),
                                                        e ? make_float2(nc.z, nc.w) : make_float2(nc.x, nc.y), ev);
                                const uint32_t wb = pack_bf16x2(wc.x, wc.y);
                                const float2 wr2 = make_float2(bf16_lo(wb), bf16_hi(wb));
                                if (e) dc1 = fadd2(dc1, wr2);
                                else dc0 = fadd2(dc0, wr2);
                                wall[i][s >> 1] = wb;
                            }
                        }
                    }
                    sT[hf * 128 + r] = tmax;
                    pair_sync(q);   // both threads' S_c and W_p reads precede any write to them
                    tmax = fmaxf(sT[r], sT[128 + r]);
                    const bool up = attempt == 0 && tmax > kRescale;
                    if (!__any_sync(0xffffffffu, up)) break;
                    // (rare) The TMEM accesses are warp-collective: rows that keep
                    // their shift take factor 1.
                    const int kup = up ? (int)ceilf(fminf(tmax, 1.0e6f)) : 0;
                    const float f = exp2_neg_int(kup);
                    m += (float)kup;
                    den *= f;
                    for (int c = 0; c < OD / 16; ++c) {   // this thread's half of O
                        float o[16];
                        tmem_ld16f(trow + p.colO + hf * OD + 16 * c, o);
                        tmem_wait_ld();
                        tmem_touch16f(o);
#pragma unroll
                        for (int i = 0; i < 16; ++i) o[i] *= f;
                        tmem_st16f(trow + p.colO + hf * OD + 16 * c, o);
                    }
                    for (int i = 0; i < 4; ++i) {         // this thread's blocks of W_p
                        const int b = 2 * i + hf;
                        if (!FULL && 16 * b >= p.M0p) break;
                        uint32_t u[8];
                        tmem_ld8(trow + p.colWp + 8 * b, u);
                        tmem_wait_ld();
                        touch8u(u);
#pragma unroll
                        for (int j = 0; j < 8; ++j) u[j] = pack_bf16x2(bf16_lo(u[j]) * f, bf16_hi(u[j]) * f);
                        tmem_st8(trow + p.colWp + 8 * b, u);
                    }
                    tmem_wait_st();
                    pair_sync(q);   // the partner's blocks of W_p are scaled too
                }
                // W_c goes over the chunk's S_c columns, except for the tile's last
                // chunk: that one goes over W_p (no lookup needs it any more), so
                // that the next tile's MMA1 may write the S columns while the last
                // MMA3c still reads W_c
                const uint32_t colWc = k + 1 == nchunks ? p.colWp : 0u;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (i >= nb) break;
                    tmem_st8(trow + colWc + 8 * (2 * i + hf), wall[i]);
                }
                den += (dc0.x + dc0.y) + (dc1.x + dc1.y);
                tmem_wait_st();
                tc_fence_before();
                if (wg_sync_or(!ok)) { failed = true; break; }
                if (leader) {   // MMA3c O += W_c x mean_child (the last chunk's W_c is over W_p)
                    tc_fence_after();
                    // after the last chunk every S column of this tile has been read
                    // and no contraction left reads one: the next tile's MMA1 first
                    if (k + 1 == nchunks && chain_next) {
                        if (issue_mma1(g + 1, stage ^ 1)) mma1_chained = true;
                        else ok = false;   // (seen by everyone at the next barrier)
                    }
                    for (int ks = 0; ks < N2 / 16; ++ks)
                        mma_ts(tmem + p.colO, tmem + colWc + 8 * ks, desc_mn(sMC, ks), idesc3, 1);
                    mma_commit(k + 1 < nchunks ? bC : bO);
                }
                __syncwarp();
            }
            if (failed) break;
        } else {
            if (wg_sync_or(!ok)) { failed = true; break; }
            if (leader) {   // MMA3p O = W_p x mean_par, the tile's only value contraction
                tc_fence_after();
                if (chain_next) {   // (S_p is read: the next tile's MMA1 first)
                    if (issue_mma1(g + 1, stage ^ 1)) mma1_chained = true;
                    else ok = false;
                }
                for (int ks = 0; ks < p.M0p / 16; ++ks)
                    mma_ts(tmem + p.colO, tmem + p.colWp + 8 * ks, desc_mn(sMP, ks), idesc3, ks > 0);
                mma_commit(bO);
            }
            __syncwarp();
        }
        pend = true;
        pend_t = t;
        pend_bh = bh;
        pend_den = den;
    }
    if (!failed && pend && epilogue(pend_t, pend_bh, pend_den)) failed = true;
    cp_async_wait_all();
    if (store_thread) bulk_wait_all();

    if (failed && tid == 0) {
        atomicExch(&p.status->error, (int)AVQ_ETIMEOUT);
        atomicExch(&p.status->where, (int)blockIdx.x);
    }
    if (failed && leader) {
        // contractions and loads still in flight finish before the TMEM and the
        // shared memory go back (each wait bounded)
        mma_commit(bFin);
        mbar_wait(bFin, 0);
        for (int st = 0; st < 2; ++st)
            if (q_pending & (1u << st)) mbar_wait(&bQ[st], (qph >> st) & 1u);
        if (head_pending) mbar_wait(bHead, hph);
        if (gat_pending) mbar_wait(bGatT, gtph);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, p.ncols);
    }
}

size_t tree_smem(int D, int M0, int C) {
    // 1 KB alignment, six [128 x D] images, 18 x 128 words of tables, the
    // mbarriers, 4 words, the child counts of one (b,h)
    return 1024 + 6 * (size_t)(D / 64) * kRegion + 128 * 4 * 18 + kBars * 8 + 16 + (size_t)M0 * C * 4;
}

template <int D, int C>
cudaError_t launch_tree(const avq_shape& s, const void* Q, const void* cb, const int32_t* counts, int P, float scale,
                        void* O, int32_t* selected, const void* means, StatusBlock* status, cudaStream_t st) {
    constexpr int MINB = D == 64 ? 2 : 1;
    const int BH = s.B * s.H;
    const int Mtot = s.M0 * (1 + s.C);
    const int M0p = (s.M0 + 15) & ~15;
    CUtensorMap tq, to, tcb, tmn, tcbc, tmnc;
    if (!make_tma_bf16_3d(&tq, Q, D, s.N, BH, kTile) || !make_tma_bf16_3d(&to, O, D, s.N, BH, kTile) ||
        !make_tma_bf16_3d(&tcb, cb, D, Mtot, s.H, M0p) || !make_tma_bf16_3d(&tmn, means, D, Mtot, BH, M0p) ||
        !make_tma_bf16_3d(&tcbc, cb, D, Mtot, s.H, C) || !make_tma_bf16_3d(&tmnc, means, D, Mtot, BH, C))
        return cudaErrorInvalidValue;
    TreeParams prm;
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
    prm.colO = 128;
    prm.colWp = 128 + D;
    prm.ncols = D == 64 ? 256 : 512;
    prm.counts = counts;
    prm.codebook = static_cast<const uint16_t*>(cb);
    prm.means = static_cast<const uint16_t*>(means);
    prm.selected = selected;
    prm.status = status;
    prm.fail_first_wait = g_fail_next_wait.exchange(0);
    const size_t smem = tree_smem(D, s.M0, C);
    const bool full = M0p == 128;
    auto kern = full ? attention_tree_kernel<D, C, MINB, true> : attention_tree_kernel<D, C, MINB, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(prm.total_tiles, sms * MINB);
    kern<<<grid, kThreads, smem, st>>>(tq, to, tcb, tmn, tcbc, tmnc, prm);
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
                                const float* vsum, int P, float scale, void* O, int32_t* selected, void* means,
                                StatusBlock* status, cudaStream_t st) {
    cudaError_t e = launch_means_bf16(vsum, counts, means, (size_t)s.B * s.H * s.M0 * (1 + s.C), s.d, st);
    if (e != cudaSuccess) return e;
#define AVQ_TREE_CASE(DD, CC) \
    if (s.d == DD && s.C == CC) return launch_tree<DD, CC>(s, Q, cb, counts, P, scale, O, selected, means, status, st);
    AVQ_TREE_CASE(64, 1) AVQ_TREE_CASE(64, 2) AVQ_TREE_CASE(64, 4) AVQ_TREE_CASE(64, 8) AVQ_TREE_CASE(64, 16)
    AVQ_TREE_CASE(128, 1) AVQ_TREE_CASE(128, 2) AVQ_TREE_CASE(128, 4) AVQ_TREE_CASE(128, 8) AVQ_TREE_CASE(128, 16)
#undef AVQ_TREE_CASE
    return cudaErrorInvalidValue;
}

}  // namespace avq

extern "C" int avq_test_fail_next_wait(void) {
    avq::g_fail_next_wait.store(1);
    return AVQ_OK;
}
