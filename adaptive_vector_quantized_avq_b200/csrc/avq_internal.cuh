// avq_internal.cuh -- definitions shared by the CUDA translation units of
// libavq_b200 (not part of the public ABI; see include/avq.h for that).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/avq.h"

namespace avq {

// Limits of the on-chip designs (checked by the entry points).
constexpr int kMaxM0 = 128;
constexpr int kMaxC = 16;
constexpr int kMaxFlat = 512;   // codewords of a flat codebook (C == 0)

// Workspace layout: the first 256 bytes are the status block.
struct StatusBlock {
    int32_t error;       // 0, or a negative avq_status set by a kernel
    int32_t where;       // kernel-specific detail (site of a timeout)
    int32_t pad[62];
};
static_assert(sizeof(StatusBlock) == 256, "status block is 256 bytes");
constexpr size_t kStatusBytes = 256;

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Host-side count of kernels enqueued by the library (avq_kernel_launches).
void count_launch(int n = 1);

// Validation of the problem sizes shared by every entry point: AVQ_OK,
// AVQ_EINVAL (null, sizes out of range) or AVQ_EUNSUPPORTED (beyond the
// kernels' on-chip limits or index arithmetic).
int check_shape(const avq_shape* s);

// ---------------------------------------------------------------- element io
__device__ __forceinline__ float ld_f32(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_f32(const __nv_bfloat16* p) {
    unsigned short u = __ldg(reinterpret_cast<const unsigned short*>(p));
    return __uint_as_float(static_cast<unsigned>(u) << 16);
}
__device__ __forceinline__ double ld_f64(const float* p) { return static_cast<double>(__ldg(p)); }
__device__ __forceinline__ double ld_f64(const __nv_bfloat16* p) {
    return static_cast<double>(ld_f32(p));
}
__device__ __forceinline__ void st_elem(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_elem(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// --------------------------------------------------------- exact decisions
// Squared distance in fp64, terms in index order, each operation rounded
// separately (no fused multiply-add): the value an fp64 reference summing
// (k_j - c_j)^2 in index order obtains, bit for bit.
template <typename T>
__device__ __noinline__ double exact_sq_dist(const T* k, const T* c, int d) {
    double s = 0.0;
    for (int j = 0; j < d; ++j) {
        double t = __dsub_rn(ld_f64(k + j), ld_f64(c + j));
        s = __dadd_rn(s, __dmul_rn(t, t));
    }
    return s;
}

// Relative error bound of an fp32 squared distance sum_j fma(t_j, t_j, acc)
// with t_j = fl(k_j - c_j): every term is non-negative, so the computed value
// lies within (d+2)u of the exact one (u = 2^-24), to first order. The
// separation test also absorbs the fp64 reference's own rounding, (d+2)2^-53.
// Two approximate distances a <= b are ordered for certain when
// b - a > eps * (a + b) + tiny.
__host__ __device__ inline float dist_eps(int d) {
    return static_cast<float>((d + 4) * (5.9604644775390625e-08 + 1.1102230246251565e-16) * 1.0625);
}
constexpr float kDistTiny = 1e-30f;

__device__ __forceinline__ bool separated(float a, float b, float eps) {
    return (b - a) > eps * (a + b) + kDistTiny;
}

}  // namespace avq
