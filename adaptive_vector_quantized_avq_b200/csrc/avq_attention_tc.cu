// avq_attention_tc.cu -- tensor-core (tcgen05) kernel of avq_attention for
// bf16 inputs, 128-query tiles (paper §4.3; papernotes, Key Designs 3).
//
// Persistent: CTAs of 256 threads walk contiguous ranges of query tiles
// (head-major, so a head's parent tables are loaded once per head). Threads r
// and r + 128 share query row r of the tile (TMEM lane r), each with half of
// the parent columns, child slots and output dimensions.
//
// Weights are kept in log-count form: for parent p the row works with
// x_p = scale*log2(e)*S_p + log2(n_p) (log2 0 = -inf), so that
// e'_p = 2^(x_p - m) = A_p n_p with one common shift m = max_p x_p; the value
// contraction then uses per-codeword MEANS (vsum / n), so its weights are the
// count-weighted e'_p. Per tile:
//   1. TMA brings the Q tile (prefetched one tile ahead, two stages).
//   2. MMA1  S_p = Q C_par^T (M=128, N=M0p, K=d) -> TMEM (for the next tile
//      of the same (b,h), issued at the end of the current one).
//   3. parent pass: x_p, m, e'_p, Zbar = sum e'_p (fp32); bf16(e'_p) -> TMEM
//      (A operand of MMA3); fp32 e'_p -> TMEM; importance terms e'_p / Zbar
//      summed over the tile's rows by a warp butterfly + 4-way smem sum.
//   4. top-P by rank over 64-bit keys (importance bits, then lower index).
//   5. MMA3p  Xbar = W_par x mean_par issued at once (overlaps the gather).
//   6. per chunk of <= 128 selected children: gather codewords and means
//      (cp.async into swizzled smem), MMA2 S_c = Q C_child^T, child weight
//      (A_c - A_p) n_c = 2^(x_c - m + log2 n_c) - A_p n_c (the parent-
//      contribution replacement of the paper's DeltaA, in count-weighted
//      form), fp32 denominator correction, bf16 weights -> TMEM, MMA3c
//      accumulates into Xbar.
//   7. O = Xbar / Zbar -> bf16 -> swizzled staging -> TMA store.
// Layouts: d = 64 with P*C <= 128 uses 256 TMEM columns (S_c aliases S_p,
// W_c aliases W_p) and ~105 KB of shared memory, so two CTAs share an SM;
// otherwise 512 columns and one CTA per SM.
#include <algorithm>

#include "avq_internal.cuh"
#include "avq_sm100.cuh"

namespace avq {
using namespace sm100;

namespace {

constexpr int kTile = 128;
constexpr uint32_t kRegion = 128 * 128;          // one 64-column block of a 128-row image
constexpr float kRangeLog2 = 86.56170245333781f;  // 60 / ln 2

struct TcAttnParams {
    int BH, H, N, M0, M0p, C, P, Mtot, ntiles, total_tiles;
    float sl2;                                    // scale * log2(e)
    uint32_t colSc, colW, colWc, colO, ncols;     // TMEM layout (S_p at column 0)
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
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
// Three-input fp32 maximum (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// One butterfly level over 2H values: lanes with `up` keep the upper half and
// send the lower one, the others the reverse; each kept value adds its
// partner's (pairs of adds packed).
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

// Sum of each of 64 columns over the 32 lanes of a warp (a butterfly that
// halves the number of values each step): on return lane L holds the sums of
// columns 2L and 2L+1 in v[0], v[1].
__device__ __forceinline__ void butterfly_colsum64(float* v, int lane) {
    butterfly_level<32>(v, lane & 16, 16);
    butterfly_level<16>(v, lane & 8, 8);
    butterfly_level<8>(v, lane & 4, 4);
    butterfly_level<4>(v, lane & 2, 2);
    butterfly_level<2>(v, lane & 1, 1);
}

// 32 TMEM columns of this warp's lanes into v (one wait for both loads).
__device__ __forceinline__ void tmem_ld32f(uint32_t taddr, float* v) {
    tmem_ld16f(taddr, v);
    tmem_ld16f(taddr + 16, v + 16);
    tmem_wait_ld();
    tmem_touch16f(v);
    tmem_touch16f(v + 16);
}

// The number of keys among k32[c0 .. c0+63] larger than parent r's in the
// order (key, complement of the index): ties go to the lower index. Not
// inlined: it runs only for tiles whose leading ranks tie.
__device__ __noinline__ int count_larger_keys64(const uint32_t* k32, int c0, uint32_t kr, int r) {
    const unsigned long long key = ((unsigned long long)kr << 32) | (uint32_t)(0xFFFFFFFFu - r);
    int rk = 0;
    for (int q = 0; q < 64; ++q) {
        const unsigned long long kq = ((unsigned long long)k32[c0 + q] << 32) | (uint32_t)(0xFFFFFFFFu - (c0 + q));
        rk += kq > key;
    }
    return rk;
}

// pair barrier: the two warps (w and w+4) that share TMEM lanes 32w..32w+31
__device__ __forceinline__ void pair_sync(int quarter) {
    asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");
}

template <int D, int C, int MINB>
__global__ void __launch_bounds__(256, MINB)
attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                    const __grid_constant__ CUtensorMap tmCB, const __grid_constant__ CUtensorMap tmMN,
                    const TcAttnParams p) {
    constexpr int KH = D / 64;
    constexpr uint32_t IMG = KH * kRegion;           // bytes of one [128 x D] bf16 image
    constexpr int KSTEPS = D / 16;
    constexpr int PPB = 32 / C;                      // selected parents behind a 32-slot block
    constexpr int OD = D / 2;                        // output dimensions per half
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align1024(smem_raw);
    uint8_t* const sQ0 = base;                       // two Q stages: sQ0, sQ0 + IMG
    uint8_t* sB1 = base + 2 * IMG;                   // parent codewords (K-major)
    uint8_t* sB3P = base + 3 * IMG;                  // parent means (MN-major)
    uint8_t* sB2 = base + 4 * IMG;                   // child codewords (K-major); O staging
    uint8_t* sB3C = base + 5 * IMG;                  // child means (MN-major)
    float* sLb = reinterpret_cast<float*>(base + 6 * IMG);   // [128] log2 n_p (-inf if empty)
    float* sInvN = sLb + 128;                                // [128] 1 / n_p
    float* sNc = sInvN + 128;                                // [128] child counts of the chunk
    float* sLc = sNc + 128;                                  // [128] their log2 (-inf if empty)
    float* sPart = sLc + 128;                                // [4][128] importance partials
    float* sX = sPart + 512;                                 // [2][128] row exchange (max, Zbar, den)
    int* sRank = reinterpret_cast<int*>(sX + 256);           // [2][128] partial ranks
    unsigned long long* sKey = reinterpret_cast<unsigned long long*>(sRank + 256);   // [128]
    int* sSel = reinterpret_cast<int*>(sKey + 128);          // [128] selected parents
    uint64_t* bars = reinterpret_cast<uint64_t*>(sSel + 128);   // q0, q1, mma, head, mma1
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 5);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = tid & 127, hf = tid >> 7, quarter = warp & 3;
    const int g0 = (int)(((long long)blockIdx.x * p.total_tiles) / gridDim.x);
    const int g1 = (int)(((long long)(blockIdx.x + 1) * p.total_tiles) / gridDim.x);

    if (warp == 0) {
        tmem_alloc(sTmem, p.ncols);
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
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);   // TMEM lanes of this row block

    const uint32_t idesc1 = idesc_bf16_f32(128, p.M0p, false);
    const uint32_t idesc3 = idesc_bf16_f32(128, D, true);
    uint32_t qph = 0, mphase = 0, hphase = 0;   // qph: phase bit of Q stage s = bit s
    float xmax = -INFINITY;
    bool failed = false;
    int cur_bh = -1;
    // Work split of a row between its two threads: half hf owns the 16-column
    // parent blocks 2b+hf (columns 32b+16hf..+16) and the 32-slot child blocks
    // 2c+hf (slots 64c+32hf..+32), so both halves stay busy for any M0 and P*C.
    const int c0 = 64 * hf;                     // this half's keys in the rank count

    auto issue_q = [&](int g, int stage) {
        const int bh = g / p.ntiles, t = g % p.ntiles;
        mbar_arrive_expect_tx(&bars[stage], IMG);
#pragma unroll
        for (int kh = 0; kh < KH; ++kh)
            tma_load_3d(sQ0 + stage * IMG + kh * kRegion, &tmQ, &bars[stage], kh * 64, t * kTile, bh);
    };
    // (thread 0) MMA1 S_p = Q C_par^T of the tile whose Q is in stage `st`,
    // completion on bars[4]; false if its Q never arrived
    auto issue_mma1 = [&](int st) -> bool {
        const bool okq = mbar_wait(&bars[st], (qph >> st) & 1u);
        qph ^= 1u << st;
        if (okq) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks)
                mma_ss(tmem, desc_k(sQ0 + st * IMG, ks), desc_k(sB1, ks), idesc1, ks > 0);
            mma_commit(&bars[4]);
        }
        return okq;
    };
    if (tid == 0 && g0 < g1) issue_q(g0, 0);

    for (int g = g0, it = 0; g < g1; ++g, ++it) {
        const int stage = it & 1;
        const int bh = g / p.ntiles, t = g % p.ntiles, h = bh % p.H;
        const int rows = min(kTile, p.N - t * kTile);
        const bool valid = r < rows;

        // the previous tile's O store must have read the staging buffer (sB2)
        if (tid == 0) bulk_wait_read_all();

        if (bh != cur_bh) {   // head change: parent codewords, parent means, counts
            if (tid == 0) {
                mbar_arrive_expect_tx(&bars[3], 2u * KH * (uint32_t)p.M0p * 128u);
#pragma unroll
                for (int kh = 0; kh < KH; ++kh) {
                    tma_load_3d(sB1 + kh * kRegion, &tmCB, &bars[3], kh * 64, 0, h);
                    tma_load_3d(sB3P + kh * kRegion, &tmMN, &bars[3], kh * 64, 0, bh);
                }
            }
            if (tid < 128) {
                const int n = tid < p.M0 ? __ldg(p.counts + (size_t)bh * p.Mtot + tid) : 0;
                sLb[tid] = n > 0 ? __log2f((float)n) : -INFINITY;
                sInvN[tid] = n > 0 ? 1.f / (float)n : 0.f;
            }
            const bool ok = mbar_wait(&bars[3], hphase);
            hphase ^= 1;
            if (__syncthreads_or(!ok)) { failed = true; break; }
            cur_bh = bh;
        }

        // ---- MMA1: S_p = Q C_par^T, and the next tile's Q into the other stage.
        // A tile issues the next one's MMA1 when that one is in the range and of
        // the same (b,h); so this one's is issued here when it is the first of
        // the range or of its (b,h). A failed wait (here and below) is acted on
        // at the next CTA barrier, which every thread reaches.
        bool ok = true;
        if (tid == 0) {
            if (g == g0 || t == 0) ok = issue_mma1(stage);
            if (ok && g + 1 < g1) issue_q(g + 1, stage ^ 1);
        }
        // (if thread 0 could not issue MMA1, every thread's wait below times out)
        ok = mbar_wait(&bars[4], (uint32_t)it & 1u) && ok;   // one MMA1 per tile, in order
        tc_fence_after();

        // ---- parent pass over this half's 64 columns
        float x[64];
#pragma unroll
        for (int b = 0; b < 4; ++b) {   // columns at or past M0p were not written: never read them
            if (32 * b + 16 * hf + 16 <= p.M0p) {
                tmem_ld16f(trow + 32 * b + 16 * hf, x + 16 * b);
            } else {
#pragma unroll
                for (int k = 0; k < 16; ++k) x[16 * b + k] = -INFINITY;
            }
        }
        tmem_wait_ld();
#pragma unroll
        for (int b = 0; b < 4; ++b) tmem_touch16f(x + 16 * b);
        const float2 sl2v = make_float2(p.sl2, p.sl2);
        float mp0 = -INFINITY, mp1 = -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; k += 4) {
            const float4 lb = *reinterpret_cast<const float4*>(sLb + 32 * (k >> 4) + 16 * hf + (k & 15));
            const float2 a = ffma2(make_float2(x[k], x[k + 1]), sl2v, make_float2(lb.x, lb.y));
            const float2 b = ffma2(make_float2(x[k + 2], x[k + 3]), sl2v, make_float2(lb.z, lb.w));
            x[k] = a.x; x[k + 1] = a.y; x[k + 2] = b.x; x[k + 3] = b.y;
            mp0 = fmax3(mp0, a.x, a.y);
            mp1 = fmax3(mp1, b.x, b.y);
        }
        sX[hf * 128 + r] = fmaxf(mp0, mp1);
        pair_sync(quarter);
        const float m = fmaxf(sX[r], sX[128 + r]);
        pair_sync(quarter);
        const float2 negm = make_float2(-m, -m);
        float2 zp0 = make_float2(0.f, 0.f), zp1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t w[8], e[16];
#pragma unroll
            for (int k = 0; k < 16; k += 2) {
                const float2 tt = fadd2(make_float2(x[16 * c + k], x[16 * c + k + 1]), negm);
                const float2 ev = make_float2(ex2(tt.x), ex2(tt.y));   // = A_p n_p (0 for empty parents)
                x[16 * c + k] = ev.x;
                x[16 * c + k + 1] = ev.y;
                if ((k >> 1) & 1) zp1 = fadd2(zp1, ev);
                else zp0 = fadd2(zp0, ev);
                e[k] = __float_as_uint(ev.x);
                e[k + 1] = __float_as_uint(ev.y);
                w[k >> 1] = pack_bf16x2(ev.x, ev.y);
            }
            tmem_st8(trow + p.colW + 16 * c + 8 * hf, w);     // bf16 weights: A operand of MMA3
            tmem_st16(trow + 32 * c + 16 * hf, e);            // fp32 e'_p kept for the child pass
        }
        sX[hf * 128 + r] = (zp0.x + zp0.y) + (zp1.x + zp1.y);
        pair_sync(quarter);
        const float z = sX[r] + sX[128 + r];
        // importance terms e'_p / Zbar_i (zero for rows past the end)
        const float rz = valid ? 1.f / z : 0.f;
        const float2 rz2 = make_float2(rz, rz);
#pragma unroll
        for (int k = 0; k < 64; k += 2) {
            const float2 v = fmul2(make_float2(x[k], x[k + 1]), rz2);
            x[k] = v.x;
            x[k + 1] = v.y;
        }
        butterfly_colsum64(x, lane);
        // lane L now holds the row-block sums of this half's x[2L], x[2L+1], i.e.
        // of parent columns 32(L/8) + 16hf + 2(L%8) and the next one
        *reinterpret_cast<float2*>(sPart + quarter * 128 + 32 * (lane >> 3) + 16 * hf + 2 * (lane & 7)) =
            make_float2(x[0], x[1]);
        tmem_wait_st();
        tc_fence_before();
        if (__syncthreads_or(!ok)) { failed = true; break; }

        // ---- importance and top-P selection. The key of a parent is the bit
        // pattern of its importance (w >= 0 orders like its bits; padding
        // parents 0); its rank is the number of larger keys, ties to the lower
        // index. Each thread of a pair counts the strictly larger keys among
        // half of the parents with 32-bit compares; when the P leading ranks
        // are free of ties (every candidate lands on its own slot) those are
        // the ranks. Otherwise the tile is ranked again over 64-bit keys
        // (importance bits, then the complement of the index).
        {
            uint32_t* sK32 = reinterpret_cast<uint32_t*>(sKey);
            if (tid < 128) {
                const float w = (sPart[tid] + sPart[128 + tid]) + (sPart[256 + tid] + sPart[384 + tid]);
                sK32[tid] = tid < p.M0 ? __float_as_uint(w) : 0u;
            }
            __syncthreads();
            const uint32_t kr = sK32[r];
            int gt = 0;
#pragma unroll 4
            for (int q = 0; q < 64; q += 4) {
                const uint4 kk = *reinterpret_cast<const uint4*>(sK32 + c0 + q);
                gt += (kk.x > kr) + (kk.y > kr) + (kk.z > kr) + (kk.w > kr);
            }
            sRank[hf * 128 + r] = gt;
            pair_sync(quarter);   // the pair's two partial counts
            int rank = -1;
            if (tid < p.M0) {
                rank = sRank[tid] + sRank[128 + tid];
                if (rank < p.P) sSel[rank] = tid;
            }
            // a candidate that does not find itself in its slot shares its key
            const bool tie = __syncthreads_or(rank >= 0 && rank < p.P && sSel[rank] != tid);
            if (tie) {
                const int rk = count_larger_keys64(sK32, c0, kr, r);
                __syncthreads();   // every thread has read the slots it checked
                sRank[hf * 128 + r] = rk;
                pair_sync(quarter);
                rank = -1;
                if (tid < p.M0) {
                    rank = sRank[tid] + sRank[128 + tid];
                    if (rank < p.P) sSel[rank] = tid;
                }
            }
            if (rank >= 0 && rank < p.P) p.selected[((size_t)bh * p.ntiles + t) * p.P + rank] = tid;
            if (tie) __syncthreads();
        }

        // ---- parents' value contribution (overlaps the child gather)
        if (tid == 0) {
            tc_fence_after();
            for (int ks = 0; ks < p.M0p / 16; ++ks)
                mma_ts(tmem + p.colO, tmem + p.colW + 8 * ks, desc_mn(sB3P, ks), idesc3, ks > 0);
        }

        // ---- children, in chunks of <= 128 slots (this half: slots 64hf..64hf+63)
        float2 den0 = make_float2(0.f, 0.f), den1 = make_float2(0.f, 0.f);   // child corrections of the denominator
        const int PC = p.P * C;
        const int nchunks = (PC + kTile - 1) / kTile;
        for (int k = 0; k < nchunks; ++k) {
            const int s0 = k * kTile;
            const int ns = min(kTile, PC - s0);
            const int N2 = (ns + 31) & ~31;   // whole 32-slot blocks: every column read is written
            for (int idx = tid; idx < N2 * (D / 8); idx += 256) {
                const int slot = idx / (D / 8), j = idx % (D / 8);
                const uint32_t off = swz(slot, j);
                if (slot < ns) {
                    const int sg = s0 + slot;
                    const int child = p.M0 + sSel[sg / C] * C + (sg % C);
                    cp_async_16(sB2 + off, p.codebook + ((size_t)h * p.Mtot + child) * D + j * 8);
                    cp_async_16(sB3C + off, p.means + ((size_t)bh * p.Mtot + child) * D + j * 8);
                } else {
                    *reinterpret_cast<uint4*>(sB2 + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(sB3C + off) = make_uint4(0, 0, 0, 0);
                }
            }
            cp_async_commit();
            if (tid < 128) {
                float nc = 0.f;
                if (tid < ns) {
                    const int sg = s0 + tid;
                    nc = (float)__ldg(p.counts + (size_t)bh * p.Mtot + p.M0 + sSel[sg / C] * C + (sg % C));
                }
                sNc[tid] = nc;
                sLc[tid] = nc > 0.f ? __log2f(nc) : -INFINITY;
            }
            // -A_p = -e'_p / n_p of the parents behind this half's two slot
            // blocks, read before MMA2 may reuse the columns
            float nap[2][PPB];
            {
                uint32_t rr[2][PPB];
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int q = 0; q < PPB; ++q)
                        tmem_ld1(trow + sSel[min((s0 + 64 * c + 32 * hf) / C + q, p.P - 1)], rr[c][q]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int q = 0; q < PPB; ++q) {
                        tmem_touch1(rr[c][q]);
                        nap[c][q] = -__uint_as_float(rr[c][q]) *
                                    sInvN[sSel[min((s0 + 64 * c + 32 * hf) / C + q, p.P - 1)]];
                    }
            }
            cp_async_wait_all();
            fence_proxy_async_smem();
            tc_fence_before();
            if (__syncthreads_or(!ok)) { failed = true; break; }
            if (tid == 0) {
                tc_fence_after();
                const uint32_t idesc2 = idesc_bf16_f32(128, N2, false);
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks)
                    mma_ss(tmem + p.colSc, desc_k(sQ0 + stage * IMG, ks), desc_k(sB2, ks), idesc2, ks > 0);
                mma_commit(&bars[2]);
            }
            ok = mbar_wait(&bars[2], mphase) && ok;
            mphase ^= 1;
            tc_fence_after();

            // child weights (A_c - A_p) n_c with A = 2^(sl2*S - m) for this half's
            // slots, as 2^(sl2*S - m + log2 n_c) - A_p n_c (empty and padding
            // slots: 0 - A_p * 0)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int sb = 64 * c + 32 * hf;                   // first slot of this block
                if (sb >= N2) break;
                float sc[32];
                tmem_ld32f(trow + p.colSc + sb, sc);
                uint32_t w[16];
#pragma unroll
                for (int kk = 0; kk < 32; kk += 4) {
                    const float4 lc = *reinterpret_cast<const float4*>(sLc + sb + kk);
                    const float4 nc = *reinterpret_cast<const float4*>(sNc + sb + kk);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int j = kk + 2 * e;                  // slot within the block
                        float2 tt = ffma2(make_float2(sc[j], sc[j + 1]), sl2v, negm);
                        tt = fadd2(tt, e ? make_float2(lc.z, lc.w) : make_float2(lc.x, lc.y));
                        xmax = fmax3(xmax, tt.x, tt.y);
                        // (past the range bound the weight may overflow: the call reports
                        // AVQ_ERANGE, and the output is not meaningful)
                        const float2 ev = make_float2(ex2(tt.x), ex2(tt.y));
                        const float2 wc = ffma2(make_float2(nap[c][j / C], nap[c][(j + 1) / C]),
                                                e ? make_float2(nc.z, nc.w) : make_float2(nc.x, nc.y), ev);
                        if (e) den1 = fadd2(den1, wc);
                        else den0 = fadd2(den0, wc);
                        w[j >> 1] = pack_bf16x2(wc.x, wc.y);
                    }
                }
                tmem_st16(trow + p.colWc + (sb >> 1), w);
            }
            tmem_wait_st();
            tc_fence_before();
            if (__syncthreads_or(!ok)) { failed = true; break; }
            if (tid == 0) {
                tc_fence_after();
                for (int ks = 0; ks < N2 / 16; ++ks)
                    mma_ts(tmem + p.colO, tmem + p.colWc + 8 * ks, desc_mn(sB3C, ks), idesc3, 1);
                mma_commit(&bars[2]);
                // every S column has been read: the next tile's MMA1 may write them
                if (k == nchunks - 1 && g + 1 < g1 && t + 1 < p.ntiles) issue_mma1(stage ^ 1);
            }
            // (each thread's own wait also orders the next chunk's writes of
            // the staging buffers and weight columns after this MMA3)
            ok = mbar_wait(&bars[2], mphase) && ok;
            mphase ^= 1;
            tc_fence_after();
        }
        if (failed) break;
        if (nchunks == 0) {   // P == 0: only the parents' contribution
            if (tid == 0) {
                mma_commit(&bars[2]);
                if (g + 1 < g1 && t + 1 < p.ntiles) issue_mma1(stage ^ 1);
            }
            ok = mbar_wait(&bars[2], mphase) && ok;
            mphase ^= 1;
            tc_fence_after();
        }

        // ---- epilogue: O = Xbar / Zbar -> bf16 -> swizzled staging -> TMA store
        sX[hf * 128 + r] = (den0.x + den0.y) + (den1.x + den1.y);
        pair_sync(quarter);
        const float inv = 1.f / (z + (sX[r] + sX[128 + r]));
        const float2 inv2 = make_float2(inv, inv);
#pragma unroll
        for (int c = 0; c < OD / 32; ++c) {
            float o[32];
            tmem_ld32f(trow + p.colO + hf * OD + 32 * c, o);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t uu[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 v = fmul2(make_float2(o[8 * q + 2 * i], o[8 * q + 2 * i + 1]), inv2);
                    uu[i] = pack_bf16x2(v.x, v.y);
                }
                const uint4 u = make_uint4(uu[0], uu[1], uu[2], uu[3]);
                *reinterpret_cast<uint4*>(sB2 + swz(r, hf * (OD / 8) + 4 * c + q)) = u;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok)) { failed = true; break; }
        if (tid == 0) {
#pragma unroll
            for (int kh = 0; kh < KH; ++kh) tma_store_3d(&tmO, sB2 + kh * kRegion, kh * 64, t * kTile, bh);
            bulk_commit();
        }
    }

    if (xmax > kRangeLog2) atomicExch(&p.status->error, (int)AVQ_ERANGE);
    if (failed && tid == 0) {
        atomicExch(&p.status->error, (int)AVQ_ETIMEOUT);
        atomicExch(&p.status->where, (int)blockIdx.x);
    }
    if (tid == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, p.ncols);
    }
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
// cancels in O = Xbar / Zbar. Two CTAs of 256 threads per SM; threads r and
// r + 128 share query row r, each with half of every chunk.
template <int D>
__global__ void __launch_bounds__(256, 2)
flat_attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                      const __grid_constant__ CUtensorMap tmCB, const __grid_constant__ CUtensorMap tmMN,
                      const TcAttnParams p) {
    static_assert(D == 64, "one 64-column block per row");
    constexpr uint32_t IMG = kRegion;
    constexpr int KSTEPS = D / 16;
    constexpr int OD = D / 2;
    constexpr uint32_t colW = 128, colO = 192;               // TMEM: S 0..127, W 128..191, O 192..255
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
        tmem_alloc(sTmem, 256);
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
        tma_load_3d(sQ, &tmQ, barQ, 0, t * kTile, bh);
    };
    // chunk c of this CTA's sequence (tile g0 + c / nch, codewords 128 (c % nch) ..) into stage c & 1
    auto issue_chunk = [&](int c) {
        const int g = g0 + c / nch, j = c % nch;
        const int bh = g / p.ntiles;
        uint64_t* bar = &barC[c & 1];
        mbar_arrive_expect_tx(bar, 2 * IMG);
        tma_load_3d(sCW + (c & 1) * IMG, &tmCB, bar, 0, 128 * j, bh % p.H);
        tma_load_3d(sMN + (c & 1) * IMG, &tmMN, bar, 0, 128 * j, bh);
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
            tma_store_3d(&tmO, sStage, 0, t * kTile, bh);
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
        tmem_dealloc(tmem, 256);
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

template <int D, int C, int MINB>
cudaError_t launch_tc(const avq_shape& s, const void* Q, const void* cb, const int32_t* counts, int P,
                      float scale, void* O, int32_t* selected, const void* means, StatusBlock* status,
                      cudaStream_t st) {
    const int BH = s.B * s.H;
    const int Mtot = s.M0 * (1 + s.C);
    const int M0p = (s.M0 + 15) & ~15;
    CUtensorMap tq, to, tcb, tmn;
    if (!make_tma_bf16_3d(&tq, Q, D, s.N, BH, kTile) || !make_tma_bf16_3d(&to, O, D, s.N, BH, kTile) ||
        !make_tma_bf16_3d(&tcb, cb, D, Mtot, s.H, M0p) || !make_tma_bf16_3d(&tmn, means, D, Mtot, BH, M0p))
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
    if (MINB == 2) {   // S_c aliases S_p, W_c aliases W_p
        prm.colSc = 0; prm.colW = 128; prm.colWc = 128; prm.colO = 192; prm.ncols = 256;
    } else {
        prm.colSc = 128; prm.colW = 256; prm.colWc = 320; prm.colO = 384; prm.ncols = 512;
    }
    prm.counts = counts;
    prm.codebook = static_cast<const uint16_t*>(cb);
    prm.means = static_cast<const uint16_t*>(means);
    prm.selected = selected;
    prm.status = status;
    const size_t need = 1024 + 6 * (size_t)(D / 64) * kRegion + 8192 + 64;
    // with 512 TMEM columns per CTA at most one CTA may be resident per SM:
    // then ask for more than half of the SM's shared memory
    const size_t smem = MINB == 2 ? need : std::max<size_t>(need, 120 * 1024);
    auto kern = attention_tc_kernel<D, C, MINB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(prm.total_tiles, sms * MINB);
    kern<<<grid, 256, smem, st>>>(tq, to, tcb, tmn, prm);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

size_t flat_attn_smem(int D, int M0) {
    const size_t M0c = (size_t)((M0 + 127) & ~127);
    return 1024 + 6 * (size_t)(D / 64) * kRegion + M0c * 4 + 768 * 4 + 5 * 8 + 16;
}

bool flat_attention_supported(const avq_shape& s, int P, int tile) {
    return s.dtype == AVQ_BF16 && s.d == 64 && s.C == 0 && P == 0 && tile == kTile && s.M0 <= 512 &&
           flat_attn_smem(s.d, s.M0) <= 227 * 1024;
}

cudaError_t launch_flat_attention(const avq_shape& s, const void* Q, const void* cb, const int32_t* counts,
                                  const float* vsum, float scale, void* O, void* means, StatusBlock* status,
                                  cudaStream_t st) {
    constexpr int D = 64;
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
    kern<<<std::min(prm.total_tiles, 2 * sms), 256, smem, st>>>(tq, to, tcb, tmn, prm);
    count_launch();
    return cudaGetLastError();
}

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
                                void* means, StatusBlock* status, cudaStream_t st) {
    const size_t nrows = (size_t)s.B * s.H * s.M0 * (1 + s.C);
    const int d4 = s.d / 4;
    means_bf16_kernel<<<(unsigned)std::min<size_t>((nrows * d4 + 255) / 256, 4096), 256, 0, st>>>(
        reinterpret_cast<const float4*>(vsum), counts, reinterpret_cast<uint2*>(means), nrows, d4);
    count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const bool small = s.d == 64 && P * s.C <= kTile;
#define AVQ_TC_CASE(DD, CC)                                                                                \
    if (s.d == DD && s.C == CC) {                                                                          \
        if (DD == 64 && small) return launch_tc<DD, CC, 2>(s, Q, cb, counts, P, scale, O, selected, means, \
                                                            status, st);                                   \
        return launch_tc<DD, CC, 1>(s, Q, cb, counts, P, scale, O, selected, means, status, st);           \
    }
    AVQ_TC_CASE(64, 1) AVQ_TC_CASE(64, 2) AVQ_TC_CASE(64, 4) AVQ_TC_CASE(64, 8) AVQ_TC_CASE(64, 16)
    AVQ_TC_CASE(128, 1) AVQ_TC_CASE(128, 2) AVQ_TC_CASE(128, 4) AVQ_TC_CASE(128, 8) AVQ_TC_CASE(128, 16)
#undef AVQ_TC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace avq
