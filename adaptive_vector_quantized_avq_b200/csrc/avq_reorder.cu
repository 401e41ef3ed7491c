// avq_reorder.cu -- query reordering along a Gilbert space-filling curve
// (paper §4.2, "Per-query-tile amortization and adaptivity"; appendix
// "Spatial reordering ablation", Table 8).
//
// avq_gilbert_order (host) lists the cells of a rows x cols token grid along
// the Gilbert curve, the generalisation of the Hilbert curve to rectangles of
// any size: the rectangle is cut recursively, into two halves along its long
// side when it is much longer than wide, else into three parts (the first
// half of its short side with the axes swapped, then the rest of the
// rectangle along its long side, then back along the second half) with the
// cut points moved by one cell where that keeps the parts' sides even, so
// that the parts' curves join end to end. Rectangles one cell thin are walked
// straight. Here the recursion is an explicit stack of pending rectangles.
//
// avq_gather_rows (device) applies such an order (or its inverse) to the rows
// of a [B,H,N,d] tensor: one thread per 16-byte chunk of a destination row.
#include <algorithm>
#include <cstdlib>
#include <vector>

#include "avq_internal.cuh"

namespace avq {
namespace {

// A pending rectangle: corner (x, y), long axis (ax, ay) and short axis
// (bx, by) as signed vectors along the grid (one of each pair is 0); its
// curve starts at the corner.
struct Rect {
    int x, y, ax, ay, bx, by;
};

int sgn(int v) { return (v > 0) - (v < 0); }
// floor(v / 2) for either sign
int half_down(int v) { return v >= 0 ? v / 2 : -((1 - v) / 2); }

__global__ void gather_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                   const int32_t* __restrict__ perm, long long rows, int N, int chunks) {
    const long long total = rows * chunks;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long row = i / chunks;
        const int c = (int)(i % chunks);
        const long long bh = row / N;
        const int n = (int)(row % N);
        const int from = __ldg(perm + n);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (from >= 0 && from < N) v = __ldg(src + (bh * N + from) * chunks + c);
        dst[i] = v;
    }
}

}  // namespace
}  // namespace avq

using namespace avq;

extern "C" int avq_gilbert_order(int rows, int cols, int32_t* order) {
    if (!order || rows < 1 || cols < 1 || (long long)rows * cols >= (1LL << 31)) return AVQ_EINVAL;
    std::vector<Rect> todo;   // the next rectangle to fill is at the back
    todo.push_back(cols >= rows ? Rect{0, 0, cols, 0, 0, rows} : Rect{0, 0, 0, rows, cols, 0});
    long long k = 0;
    while (!todo.empty()) {
        const Rect r = todo.back();
        todo.pop_back();
        const int w = std::abs(r.ax + r.ay), h = std::abs(r.bx + r.by);
        const int ux = sgn(r.ax), uy = sgn(r.ay), vx = sgn(r.bx), vy = sgn(r.by);
        if (h == 1 || w == 1) {   // one cell thin: walk it
            const int n = h == 1 ? w : h, sx = h == 1 ? ux : vx, sy = h == 1 ? uy : vy;
            for (int i = 0, x = r.x, y = r.y; i < n; ++i, x += sx, y += sy) order[k++] = y * cols + x;
            continue;
        }
        int ax2 = half_down(r.ax), ay2 = half_down(r.ay), bx2 = half_down(r.bx), by2 = half_down(r.by);
        if (2 * w > 3 * h) {
            // much longer than wide: the two halves of the long side, the
            // first made even where possible
            if ((std::abs(ax2 + ay2) & 1) && w > 2) { ax2 += ux; ay2 += uy; }
            todo.push_back({r.x + ax2, r.y + ay2, r.ax - ax2, r.ay - ay2, r.bx, r.by});
            todo.push_back({r.x, r.y, ax2, ay2, r.bx, r.by});
        } else {
            // three parts (pushed last first): along the first half of the
            // short side with the axes swapped, then the remaining rectangle
            // along the long side, then back along the second half of the
            // long side, ending next to the start's long edge
            if ((std::abs(bx2 + by2) & 1) && h > 2) { bx2 += vx; by2 += vy; }
            todo.push_back({r.x + (r.ax - ux) + (bx2 - vx), r.y + (r.ay - uy) + (by2 - vy), -bx2, -by2,
                            -(r.ax - ax2), -(r.ay - ay2)});
            todo.push_back({r.x + bx2, r.y + by2, r.ax, r.ay, r.bx - bx2, r.by - by2});
            todo.push_back({r.x, r.y, bx2, by2, ax2, ay2});
        }
    }
    return k == (long long)rows * cols ? AVQ_OK : AVQ_EINVAL;
}

extern "C" int avq_gather_rows(const avq_shape* s, const void* src, void* dst, const int32_t* perm,
                               void* stream) {
    if (!s || s->B < 1 || s->H < 1 || s->N < 0 || (s->d != 64 && s->d != 128)) return AVQ_EINVAL;
    if (s->dtype != AVQ_F32 && s->dtype != AVQ_BF16) return AVQ_EINVAL;
    if ((long long)s->B * s->H * s->N * s->d >= (1LL << 40)) return AVQ_EUNSUPPORTED;
    if (s->N == 0) return AVQ_OK;
    const auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
    if (!src || !dst || !perm || !al(src, 16) || !al(dst, 16) || !al(perm, 4)) return AVQ_EINVAL;
    const int chunks = s->d * (s->dtype == AVQ_BF16 ? 2 : 4) / 16;
    const long long rows = (long long)s->B * s->H * s->N;
    const long long total = rows * chunks;
    const unsigned blocks = (unsigned)std::min<long long>((total + 255) / 256, 148LL * 32);
    gather_rows_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), perm, rows, s->N, chunks);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? AVQ_OK : AVQ_ECUDA;
}
