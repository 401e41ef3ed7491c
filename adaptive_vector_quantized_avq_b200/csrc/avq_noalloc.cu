// avq_noalloc.cu -- avq_attention_noalloc: the attention call for callers
// that cannot allocate device memory.
//
// avq_attention needs a caller-provided workspace: a status word plus a bf16
// copy of the value sums that the tensor-core kernel reads. Some callers
// cannot provide one: a host framework that owns every device allocation
// and forbids its plugins to call cudaMalloc, or latency-bound code for which
// cudaMalloc (which can synchronise the device) is not acceptable on the hot
// path. This entry point keeps that scratch in a fixed array of device memory
// that belongs to the library, so the caller passes only inputs and outputs.
//
// The array is kNoAllocScratchBytes (8 MiB) of global memory on every GPU that
// loads the library, held until the process exits. A problem whose scratch
// (256 bytes + B*H*M0*(1+C)*d*2 bytes) does not fit is rejected with
// AVQ_EWORKSPACE. All calls on a device share the array: calls whose work
// overlaps on the GPU (other streams, other host threads) race on it and must
// be serialised by the caller.
#include <mutex>

#include "avq_internal.cuh"

namespace avq {
bool attention_tc_supported(const avq_shape& s, int tile);
size_t attention_tc_workspace(const avq_shape& s);
cudaError_t launch_attention_tc(const avq_shape& s, const void* Q, const void* cb, const int32_t* counts,
                                const float* vsum, int P, float scale, void* O, int32_t* selected,
                                void* vtab, StatusBlock* status, cudaStream_t st);
cudaError_t launch_attention_simt(const avq_shape& s, const void* Q, const void* cb,
                                  const int32_t* counts, const float* vsum, int P, int tile,
                                  float scale, void* O, int32_t* selected, cudaStream_t st);
}  // namespace avq

using namespace avq;

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB
constexpr int kMaxDevices = 64;

// The scratch. In host code this name is only a stand-in for the symbol; the
// device address comes from cudaGetSymbolAddress (see scratch_for_device).
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device; looked up once per
// device, with that device current, on the first call there.
cudaError_t scratch_for_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int avq_attention_noalloc(const avq_shape* s, const void* Q, const void* codebook,
                                     const int32_t* counts, const float* vsum, int P, int tile, float scale,
                                     void* O, int32_t* selected, int32_t* device_status, void* stream) {
    const int rc = check_shape(s);   // the same size checks as every entry point
    if (rc != AVQ_OK) return rc;
    if (s->C == 0) return AVQ_EUNSUPPORTED;   // flat codebooks: avq_attention
    if (P < 0 || P > s->M0 || (tile != 64 && tile != 128)) return AVQ_EINVAL;
    if (!(scale > 0.f) || !(scale < 3.0e38f)) return AVQ_EINVAL;
    if (!codebook || !counts || !vsum) return AVQ_EINVAL;
    if (s->N > 0 && (!Q || !O || (P > 0 && !selected))) return AVQ_EINVAL;
    if (!aligned_to(Q, 16) || !aligned_to(O, 16) || !aligned_to(codebook, 16) || !aligned_to(vsum, 16) ||
        !aligned_to(counts, 4) || !aligned_to(selected, 4) || !aligned_to(device_status, 4))
        return AVQ_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool tc = attention_tc_supported(*s, tile);
    if (tc && kStatusBytes + attention_tc_workspace(*s) > kNoAllocScratchBytes) return AVQ_EWORKSPACE;
    if (s->N == 0) {
        if (device_status && cudaMemsetAsync(device_status, 0, sizeof(int32_t), st) != cudaSuccess) return AVQ_ECUDA;
        return AVQ_OK;
    }
    cudaError_t e;
    if (tc) {
        void* scratch = nullptr;
        if (scratch_for_device(&scratch) != cudaSuccess) return AVQ_ECUDA;
        uint8_t* base = static_cast<uint8_t*>(scratch);
        // the status word must start at zero; the value table is fully rewritten
        if (cudaMemsetAsync(base, 0, kStatusBytes, st) != cudaSuccess) return AVQ_ECUDA;
        e = launch_attention_tc(*s, Q, codebook, counts, vsum, P, scale, O, selected, base + kStatusBytes,
                                reinterpret_cast<StatusBlock*>(base), st);
        if (e == cudaSuccess && device_status)
            e = cudaMemcpyAsync(device_status, base, sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
    } else {
        // this shape runs on the CUDA-core kernel, which needs no scratch
        e = launch_attention_simt(*s, Q, codebook, counts, vsum, P, tile, scale, O, selected, st);
        if (e == cudaSuccess && device_status) e = cudaMemsetAsync(device_status, 0, sizeof(int32_t), st);
    }
    return e == cudaSuccess ? AVQ_OK : AVQ_ECUDA;
}
