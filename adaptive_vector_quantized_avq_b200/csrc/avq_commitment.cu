// avq_commitment.cu -- avq_commitment: per-(b,h) sum of the squared distance
// between each key and the codeword it is assigned to (paper, appendix
// "Per-layer codebook analysis", Table 7, commitment loss).
//
// Grid (chunks, B*H); a warp takes one key at a time, its lanes splitting the
// d coordinates (2 or 4 each): the key row and the codeword row are read
// coalesced, each lane keeps an fp64 running sum of its coordinates' squared
// differences (taken in fp32), and the block's sums meet in one fp64 atomic
// per block.
#include <algorithm>

#include "avq_internal.cuh"

namespace avq {
namespace {

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<uint16_t>(uint16_t x) { return __uint_as_float((uint32_t)x << 16); }

template <typename T, int D>
__global__ void __launch_bounds__(256) commitment_kernel(const T* __restrict__ K, const T* __restrict__ cb,
                                                         const int32_t* __restrict__ assign, double* sq_err,
                                                         int H, int N, int Mtot) {
    constexpr int DL = D / 32;   // coordinates per lane
    __shared__ double sW[8];
    const int bh = blockIdx.y, h = bh % H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const T* kb = K + (size_t)bh * N * D;
    const T* cbh = cb + (size_t)h * Mtot * D;
    const int32_t* ab = assign + (size_t)bh * N;
    double acc = 0.0;
    for (int n = blockIdx.x * 8 + warp; n < N; n += gridDim.x * 8) {
        const int a = __ldg(ab + n);
        if (a < 0 || a >= Mtot) {
            acc = __longlong_as_double(0x7ff8000000000000LL);   // NaN: an id outside the tree
            continue;
        }
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < DL; ++e) {
            const int j = lane * DL + e;
            const float t = __fsub_rn(to_f32(__ldg(kb + (size_t)n * D + j)), to_f32(__ldg(cbh + (size_t)a * D + j)));
            s = __fmaf_rn(t, t, s);
        }
        acc += (double)s;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) sW[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < 8; ++w) t += sW[w];
        atomicAdd(sq_err + bh, t);
    }
}

template <typename T, int D>
cudaError_t launch(const avq_shape& s, const void* K, const void* cb, const int32_t* assign, double* out,
                   cudaStream_t st) {
    const int BH = s.B * s.H, Mtot = s.M0 * (1 + s.C);
    const int chunks = std::max(1, std::min((s.N + 255) / 256, 64));
    commitment_kernel<T, D><<<dim3(chunks, BH), 256, 0, st>>>(static_cast<const T*>(K), static_cast<const T*>(cb),
                                                              assign, out, s.H, s.N, Mtot);
    count_launch();
    return cudaGetLastError();
}

}  // namespace
}  // namespace avq

using namespace avq;

extern "C" int avq_commitment(const avq_shape* s, const void* K, const void* codebook, const int32_t* assign,
                              double* sq_err, void* stream) {
    if (!s) return AVQ_EINVAL;
    if (s->B < 1 || s->H < 1 || s->N < 0 || (s->d != 64 && s->d != 128)) return AVQ_EINVAL;
    if (s->dtype != AVQ_F32 && s->dtype != AVQ_BF16) return AVQ_EINVAL;
    if (s->M0 < 1 || s->C < 0) return AVQ_EINVAL;
    if (s->M0 > (s->C == 0 ? kMaxFlat : kMaxM0) || s->C > kMaxC) return AVQ_EUNSUPPORTED;
    if ((long long)s->B * s->H * s->N * s->d >= (1LL << 40) || (long long)s->B * s->H > 65535) return AVQ_EUNSUPPORTED;
    const auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
    if (!codebook || !sq_err || (s->N > 0 && (!K || !assign))) return AVQ_EINVAL;
    if (!al(K, 16) || !al(codebook, 16) || !al(assign, 4) || !al(sq_err, 8)) return AVQ_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(sq_err, 0, sizeof(double) * s->B * s->H, st) != cudaSuccess) return AVQ_ECUDA;
    if (s->N == 0) return AVQ_OK;
    cudaError_t e;
    if (s->dtype == AVQ_BF16)
        e = s->d == 64 ? launch<uint16_t, 64>(*s, K, codebook, assign, sq_err, st)
                       : launch<uint16_t, 128>(*s, K, codebook, assign, sq_err, st);
    else
        e = s->d == 64 ? launch<float, 64>(*s, K, codebook, assign, sq_err, st)
                       : launch<float, 128>(*s, K, codebook, assign, sq_err, st);
    return e == cudaSuccess ? AVQ_OK : AVQ_ECUDA;
}
