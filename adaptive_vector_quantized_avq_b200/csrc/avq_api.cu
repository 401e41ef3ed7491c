// avq_api.cu -- the extern "C" entry points declared in include/avq.h:
// argument validation on the host, zeroing of outputs on the stream, and the
// choice of kernel for the shape and dtype.
#include <stdint.h>

#include <atomic>

#include <algorithm>

#include "avq_internal.cuh"

namespace avq {
static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

int check_shape(const avq_shape* s) {
    if (!s) return AVQ_EINVAL;
    if (s->B < 1 || s->H < 1 || s->N < 0) return AVQ_EINVAL;
    if (s->d != 64 && s->d != 128) return AVQ_EINVAL;
    if (s->dtype != AVQ_F32 && s->dtype != AVQ_BF16) return AVQ_EINVAL;
    if (s->M0 < 1 || s->C < 0) return AVQ_EINVAL;
    // a tree holds up to kMaxM0 parents; a flat codebook (C == 0) up to kMaxFlat codewords
    if (s->M0 > (s->C == 0 ? kMaxFlat : kMaxM0) || s->C > kMaxC) return AVQ_EUNSUPPORTED;
    // element counts must fit the kernels' index arithmetic
    const long long rows = (long long)s->B * s->H * s->N;
    if (rows * s->d >= (1LL << 40)) return AVQ_EUNSUPPORTED;
    if ((long long)s->B * s->H > 65535LL * 32) return AVQ_EUNSUPPORTED;
    return AVQ_OK;
}
}  // namespace avq

namespace avq {
cudaError_t launch_precompute_simt(const avq_shape& s, const void* K, const void* V,
                                   const void* cb, int32_t* assign, int32_t* counts,
                                   float* vsum, cudaStream_t st);
cudaError_t launch_attention_simt(const avq_shape& s, const void* Q, const void* cb,
                                  const int32_t* counts, const float* vsum, int P, int tile,
                                  float scale, void* O, int32_t* selected, cudaStream_t st);
size_t attention_simt_smem(const avq_shape& s);
bool attention_tc_supported(const avq_shape& s, int tile);
bool precompute_tc_supported(const avq_shape& s);
cudaError_t launch_precompute_tc(const avq_shape& s, const void* K, const void* V, const void* cb,
                                 int32_t* assign, int32_t* counts, float* vsum, StatusBlock* status,
                                 cudaStream_t st);
size_t attention_tc_workspace(const avq_shape& s);
bool flat_precompute_supported(const avq_shape& s);
cudaError_t launch_flat_precompute(const avq_shape& s, const void* K, const void* V, const void* cb,
                                   int32_t* assign, int32_t* counts, float* vsum, StatusBlock* status,
                                   cudaStream_t st);
bool flat_attention_supported(const avq_shape& s, int P, int tile);
cudaError_t launch_flat_attention(const avq_shape& s, const void* Q, const void* cb, const int32_t* counts,
                                  const float* vsum, float scale, void* O, void* means, StatusBlock* status,
                                  cudaStream_t st);
cudaError_t launch_attention_tc(const avq_shape& s, const void* Q, const void* cb, const int32_t* counts,
                                const float* vsum, int P, float scale, void* O, int32_t* selected,
                                void* vtab, StatusBlock* status, cudaStream_t st);
}  // namespace avq

using namespace avq;

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_ws(const void* ws, size_t have, size_t need) {
    if (need == 0) return AVQ_OK;
    if (!ws || have < need) return AVQ_EWORKSPACE;
    if (!aligned(ws, 256)) return AVQ_EINVAL;
    return AVQ_OK;
}

}  // namespace

extern "C" {

int avq_version(void) { return 100; }

uint64_t avq_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char* avq_status_string(int st) {
    switch (st) {
        case AVQ_OK: return "AVQ_OK";
        case AVQ_EINVAL: return "AVQ_EINVAL: invalid argument (null or misaligned pointer, size out of range)";
        case AVQ_EUNSUPPORTED: return "AVQ_EUNSUPPORTED: sizes beyond the on-chip limits of the kernels";
        case AVQ_ECUDA: return "AVQ_ECUDA: a CUDA call failed";
        case AVQ_ETIMEOUT: return "AVQ_ETIMEOUT: a bounded device-side wait ran out";
        case AVQ_EWORKSPACE: return "AVQ_EWORKSPACE: workspace missing or too small";
        case AVQ_ERANGE: return "AVQ_ERANGE: a weight out of range (reserved)";
        default: return "unknown avq status";
    }
}

namespace {
// Zeroes the precompute outputs that are accumulated (counts, vsum): one
// launch instead of two memsets.
__global__ void zero_accumulators_kernel(int32_t* counts, size_t n_counts, float4* vsum4, size_t n_vsum4) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t i0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (size_t i = i0; i < n_vsum4; i += stride) vsum4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (size_t i = i0; i < n_counts; i += stride) counts[i] = 0;
}
}  // namespace

size_t avq_precompute_workspace_bytes(const avq_shape* s) {
    if (check_shape(s) != AVQ_OK) return 0;
    // status block, then room to list every key whose decision the fp32
    // bounds leave open: 8 bytes per key, the last 128-key tile of each
    // sequence counted whole
    const size_t tiles = (size_t)s->B * s->H * (((size_t)s->N + 127) / 128);
    return kStatusBytes + align256(sizeof(long long) * tiles * 128);
}

int avq_precompute(const avq_shape* s, const void* K, const void* V, const void* codebook,
                   int32_t* assign, int32_t* counts, float* vsum, void* workspace,
                   size_t workspace_bytes, void* stream) {
    int rc = check_shape(s);
    if (rc != AVQ_OK) return rc;
    if (!codebook || !counts || !vsum) return AVQ_EINVAL;
    if (s->N > 0 && (!K || !V || !assign)) return AVQ_EINVAL;
    if (!aligned(K, 16) || !aligned(V, 16) || !aligned(codebook, 16) || !aligned(vsum, 16) ||
        !aligned(assign, 4) || !aligned(counts, 4))
        return AVQ_EINVAL;
    rc = check_ws(workspace, workspace_bytes, avq_precompute_workspace_bytes(s));
    if (rc != AVQ_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t Mtot = (size_t)s->M0 * (1 + s->C);
    const size_t BH = (size_t)s->B * s->H;
    if (s->C == 0 && !flat_precompute_supported(*s)) return AVQ_EUNSUPPORTED;
    const bool tc = s->N > 0 && s->C > 0 && precompute_tc_supported(*s);
    StatusBlock* status = static_cast<StatusBlock*>(workspace);
    {
        // counts and vsum start at zero
        const size_t n4 = BH * Mtot * s->d / 4;   // d is a multiple of 4
        const unsigned blocks = (unsigned)std::min<size_t>((n4 + 255) / 256, 1024);
        zero_accumulators_kernel<<<blocks > 0 ? blocks : 1, 256, 0, st>>>(
            counts, BH * Mtot, reinterpret_cast<float4*>(vsum), n4);
        count_launch();
        if (cudaGetLastError() != cudaSuccess) return AVQ_ECUDA;
    }
    if (s->N == 0) return AVQ_OK;
    cudaError_t e;
    if (s->C == 0) {
        e = launch_flat_precompute(*s, K, V, codebook, assign, counts, vsum, status, st);
    } else if (tc) {
        e = launch_precompute_tc(*s, K, V, codebook, assign, counts, vsum, status, st);
    } else {
        e = launch_precompute_simt(*s, K, V, codebook, assign, counts, vsum, st);
    }
    return e == cudaSuccess ? AVQ_OK : AVQ_ECUDA;
}

size_t avq_attention_workspace_bytes(const avq_shape* s, int P, int tile) {
    if (check_shape(s) != AVQ_OK) return 0;
    if (P < 0 || P > s->M0 || (tile != 64 && tile != 128)) return 0;
    size_t n = kStatusBytes;
    if (s->C == 0) {
        if (!flat_attention_supported(*s, P, tile)) return 0;
        n += attention_tc_workspace(*s);
    } else if (attention_tc_supported(*s, tile)) {
        n += attention_tc_workspace(*s);
    }
    return n;
}

int avq_attention(const avq_shape* s, const void* Q, const void* codebook, const int32_t* counts,
                  const float* vsum, int P, int tile, float scale, void* O, int32_t* selected,
                  void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_shape(s);
    if (rc != AVQ_OK) return rc;
    if (P < 0 || P > s->M0 || (tile != 64 && tile != 128)) return AVQ_EINVAL;
    if (s->C == 0 && P != 0) return AVQ_EINVAL;   // a flat codebook has nothing to select
    if (s->C == 0 && !flat_attention_supported(*s, P, tile)) return AVQ_EUNSUPPORTED;
    if (!(scale > 0.f) || !(scale < 3.0e38f)) return AVQ_EINVAL;
    if (!codebook || !counts || !vsum) return AVQ_EINVAL;
    if (s->N > 0 && (!Q || !O || (P > 0 && !selected))) return AVQ_EINVAL;
    if (!aligned(Q, 16) || !aligned(O, 16) || !aligned(codebook, 16) || !aligned(vsum, 16) ||
        !aligned(counts, 4) || !aligned(selected, 4))
        return AVQ_EINVAL;
    rc = check_ws(workspace, workspace_bytes, avq_attention_workspace_bytes(s, P, tile));
    if (rc != AVQ_OK) return rc;
    if (s->N == 0) return AVQ_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (s->C == 0) {
        uint8_t* ws = static_cast<uint8_t*>(workspace);
        e = launch_flat_attention(*s, Q, codebook, counts, vsum, scale, O, ws + kStatusBytes,
                                  reinterpret_cast<StatusBlock*>(ws), st);
    } else if (attention_tc_supported(*s, tile)) {
        uint8_t* ws = static_cast<uint8_t*>(workspace);
        e = launch_attention_tc(*s, Q, codebook, counts, vsum, P, scale, O, selected, ws + kStatusBytes,
                                reinterpret_cast<StatusBlock*>(ws), st);
    } else {
        e = launch_attention_simt(*s, Q, codebook, counts, vsum, P, tile, scale, O, selected, st);
    }
    return e == cudaSuccess ? AVQ_OK : AVQ_ECUDA;
}

int avq_device_status(void* workspace, void* stream) {
    if (!workspace || !aligned(workspace, 256)) return AVQ_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    StatusBlock host;
    if (cudaMemcpyAsync(&host, workspace, sizeof(host), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return AVQ_ECUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return AVQ_ECUDA;
    if (host.error != 0) {
        const int32_t zero = 0;
        if (cudaMemcpyAsync(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice, st) != cudaSuccess)
            return AVQ_ECUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return AVQ_ECUDA;
        return host.error;
    }
    return AVQ_OK;
}

}  // extern "C"
