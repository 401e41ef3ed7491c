/*
 * avq.h -- C ABI of the AVQ-attention forward path on NVIDIA B200 (sm_100a).
 *
 * AVQ-attention ("AVQ-Attention: Adaptive Vector-Quantized Attention")
 * replaces the keys of softmax attention by codewords of a frozen two-level
 * tree codebook and refines, per query tile, the most attended parents with
 * their children. The forward pass is two calls:
 *
 *   avq_precompute  -- paper §4.2 ("Vector Quantization for (A)VQ-Attention");
 *                      papernotes summary, Key Designs 2 (fused full-tree
 *                      precomputation): key assignment and per-codeword
 *                      counts and value sums for the whole tree.
 *   avq_attention   -- paper §4.3 ("Computing (A)VQ-Attention with Flash
 *                      Attention"); papernotes summary, Key Designs 3:
 *                      parent attention, codeword importance, top-P parent
 *                      selection per query tile, child attention with the
 *                      parent-contribution correction, output.
 *
 * Conventions common to every call
 * --------------------------------
 * - Pointers named "device" must point to memory of the current CUDA device;
 *   the caller owns and allocates every buffer. The library allocates no
 *   memory and never synchronises the stream: each call only enqueues work
 *   on `stream` (a cudaStream_t passed as void*; NULL is the legacy default
 *   stream) and returns.
 * - Tensors are dense, row-major, C-contiguous:
 *     K, V, Q, O : [B, H, N, d]            element type `dtype`
 *     codebook   : [H, Mtot, d]            element type `dtype`, Mtot = M0*(1+C)
 *                  tree order: parents 0..M0-1, then child c of parent p at
 *                  row M0 + p*C + c (each parent's children are contiguous,
 *                  paper §4.3 "Child spawning"); one codebook per head,
 *                  shared by the batch (paper §4.1).
 *     assign     : [B, H, N]        int32  leaf id of each key, in tree order
 *     counts     : [B, H, Mtot]     int32
 *     vsum       : [B, H, Mtot, d]  float32
 *     selected   : [B, H, ceil(N/tile), P] int32
 * - Alignment: K, V, Q, O, codebook, vsum and the workspace 16 bytes;
 *   assign, counts, selected 4 bytes.
 * - Return value: AVQ_OK (0) or a negative avq_status. Argument errors are
 *   detected on the host before anything is enqueued, and leave every output
 *   untouched. A launch failure returns AVQ_ECUDA.
 */
#ifndef AVQ_B200_H
#define AVQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of K, V, Q, O and the codebook (all the same). */
typedef enum { AVQ_F32 = 0, AVQ_BF16 = 1 } avq_dtype;

/* Problem sizes. Supported: B, H >= 1; N >= 0; d in {64, 128};
 * a tree: 1 <= M0 <= 128, 1 <= C <= 16;
 * a flat codebook (C == 0, M0 codewords and no children; paper §3.2 VQ
 * attention): 1 <= M0 <= 512, bf16 only; avq_attention then takes P == 0
 * with tile 128 (other flat cases return AVQ_EUNSUPPORTED). */
typedef struct {
    int32_t B, H, N, d;
    int32_t M0, C;
    int32_t dtype; /* avq_dtype */
} avq_shape;

typedef enum {
    AVQ_OK = 0,
    AVQ_EINVAL = -1,        /* null/misaligned pointer, size or argument out of range */
    AVQ_EUNSUPPORTED = -2,  /* sizes beyond what the kernels hold on chip (e.g. M0 > 128) */
    AVQ_ECUDA = -3,         /* a CUDA launch or runtime call failed */
    AVQ_ETIMEOUT = -4,      /* a bounded device-side wait ran out (reported by avq_device_status) */
    AVQ_EWORKSPACE = -5,    /* workspace missing or smaller than the *_workspace_bytes() answer */
    AVQ_ERANGE = -6         /* reserved (no current kernel reports it): a weight out of range */
} avq_status;

/*
 * Workspace needed by avq_precompute for `s` (bytes, a multiple of 256;
 * 0 for invalid shapes): 256 bytes for the device status word read by
 * avq_device_status, then 8 bytes per key (B*H*ceil(N/128)*128) for the list
 * of keys whose nearest parent or leaf the kernel's fp32 error bounds leave
 * open; those keys are then decided exactly (fp64) within the same call.
 */
size_t avq_precompute_workspace_bytes(const avq_shape* s);

/*
 * Fused full-tree VQ precompute (paper §4.2; papernotes, Key Designs 2;
 * paper Table 1, rows "VQ assignment" and "Value aggregation").
 *
 * For every key k of head (b,h):
 *   p*(k)  = argmin_p ||K_k - C_p||^2 over the M0 parents (squared Euclidean
 *            distance; ties to the lowest index), distance kept;
 *   leaf   = the child M0 + p*C + c of p* with the smallest distance if that
 *            distance is STRICTLY smaller than the kept parent distance
 *            (lowest c among equal children), else p*;
 *   assign[b,h,k] = leaf.
 * Decisions are those of exact fp64 arithmetic on the stored values: the
 * kernels filter with fp32 distances and a rigorous error bound and re-decide
 * in fp64 whenever the bound does not separate the candidates.
 *   counts[b,h,p] / vsum[b,h,p,:] : number / sum of V rows of ALL keys with
 *                                   p*(k) = p (the parent's whole cluster);
 *   counts[b,h,j] / vsum[b,h,j,:] : for a child j, only the keys whose leaf is j.
 * vsum is accumulated in fp32 (summation order unspecified).
 * With C == 0 the leaf is p*(k) itself: the nearest of the M0 codewords.
 *
 * K, V, codebook: device, read only. assign, counts, vsum: device, written
 * (zeroed by the call). workspace: device, >= avq_precompute_workspace_bytes(s).
 */
int avq_precompute(const avq_shape* s, const void* K, const void* V, const void* codebook,
                   int32_t* assign, int32_t* counts, float* vsum,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Workspace needed by avq_attention for `s`, P and tile (bytes, multiple of
 * 256; 0 for invalid arguments). It holds the device status word and
 * per-head tables derived from counts/vsum each call.
 */
size_t avq_attention_workspace_bytes(const avq_shape* s, int P, int tile);

/*
 * Tiled adaptive attention (paper §4.3; papernotes, Key Designs 3).
 *
 * Queries of head (b,h) are cut into consecutive tiles of `tile` rows
 * (tile in {64, 128}; a partial last tile is masked). For each query i:
 *   S_ij = scale * Q_i . C_j  (the paper writes exp(Q C^T), scale folded in Q);
 *   parent attention  A_ip = exp(S_ip - m_i), Zbar_i = sum_p A_ip n_p, over
 *   parents with n_p > 0 (m_i their largest logit).
 * For each tile I:
 *   importance w_p(I) = sum_{i in I} A_ip n_p / Zbar_i ("Codeword importance");
 *   selected[b,h,t,:] = the P parents of largest w, by descending w, ties to
 *   the lower index ("Child spawning"); 0 <= P <= M0.
 * Output, with one shift for all terms of query i:
 *   Xbar_i = sum_p e^{S_ip} vsum_p
 *          + sum_{p selected} sum_c (e^{S_ic} - e^{S_ip}) vsum_{p,c}
 *   Zbar_i likewise with counts (the DeltaA correction of papernotes, Key
 *   Designs 3);  O_i = Xbar_i / Zbar_i, stored in Q's dtype.
 * counts/vsum are avq_precompute's outputs for the same codebook.
 * With C == 0 (a flat codebook) P must be 0 (AVQ_EINVAL otherwise): O is
 * VQ attention over the M0 codewords, O_i = sum_p e^{S_ip} vsum_p / Zbar_i.
 *
 * Q, codebook, counts, vsum: device, read only. O, selected: device,
 * written. selected may be NULL when P == 0. workspace: device,
 * >= avq_attention_workspace_bytes(s, P, tile).
 */
int avq_attention(const avq_shape* s, const void* Q, const void* codebook,
                  const int32_t* counts, const float* vsum, int P, int tile, float scale,
                  void* O, int32_t* selected, void* workspace, size_t workspace_bytes,
                  void* stream);

/*
 * avq_attention for callers that cannot allocate device memory (a host
 * framework that owns all device allocations and forbids its plugins to call
 * cudaMalloc, or latency-bound code that cannot afford cudaMalloc's implicit
 * device synchronisation). The paper has no counterpart: this is a property
 * of the library's interface only. Same arguments, results and errors as
 * avq_attention for trees (C >= 1; a flat codebook, C == 0, returns
 * AVQ_EUNSUPPORTED here: use avq_attention), with no workspace: the scratch
 * lives in a fixed 8 MiB array of device memory owned by the library (on
 * every GPU that loads it, until the process exits).
 *
 * - Problems whose scratch, 256 + B*H*M0*(1+C)*d*2 bytes, exceeds 8 MiB are
 *   rejected with AVQ_EWORKSPACE before anything is enqueued.
 * - The first call on a device looks the array's device address up (once per
 *   device, with that device current); make that first call before any
 *   stream capture on the device.
 * - All calls on a device share the array and it keeps the last call's
 *   contents; calls whose work overlaps on the GPU (different streams or host
 *   threads) race on it and must be serialised by the caller.
 * - device_status (device pointer to one int32, may be NULL) receives this
 *   call's device status word (AVQ_OK or AVQ_ETIMEOUT), written
 *   on `stream`.
 * - Allocates nothing: no cudaMalloc/cudaFree and no allocating library call.
 */
int avq_attention_noalloc(const avq_shape* s, const void* Q, const void* codebook,
                          const int32_t* counts, const float* vsum, int P, int tile, float scale,
                          void* O, int32_t* selected, int32_t* device_status, void* stream);

/*
 * Commitment loss of an assignment (paper, appendix "Per-layer codebook
 * analysis", Table 7: the mean squared distance between each key and its
 * assigned codeword; here the assigned codeword is the key's leaf, as written
 * to `assign` by avq_precompute). A diagnostic, outside the forward path.
 *
 * For every (b,h): sq_err[b*H + h] = sum over n of
 *   ||K[b,h,n] - codebook[h, assign[b,h,n]]||^2
 * (divide by N for the mean). Each squared difference is taken in fp32 from
 * the stored values, the sums are accumulated in fp64 (order unspecified).
 * A leaf id outside [0, M0*(1+C)) makes its (b,h) sum NaN.
 *
 * K, codebook: device, as for avq_precompute (16-byte aligned). assign:
 * device [B,H,N] int32 (4-byte aligned). sq_err: device, B*H doubles
 * (8-byte aligned), overwritten. Returns AVQ_OK, AVQ_EINVAL (null or
 * misaligned pointer, invalid shape), AVQ_EUNSUPPORTED, AVQ_ECUDA. Does not
 * synchronise.
 */
int avq_commitment(const avq_shape* s, const void* K, const void* codebook, const int32_t* assign,
                   double* sq_err, void* stream);

/*
 * Top-P capture (paper §5.2 "Elastic Inference via Top-P Adjustment",
 * Table 6; Figure 7): for every query i of head (b,h), in tile t = i / tile,
 *   capture[b,h,i] = sum_{k : parent(k) in sel(t)} e^{s_ik} / sum_k e^{s_ik},
 *   s_ik = scale * Q_i . K_k over ALL N keys of the head (the true, exact
 *   softmax attention weights),
 * where parent(k) = assign[b,h,k] if < M0, else (assign[b,h,k] - M0) / C (the
 * leaf's parent), and sel(t) = selected[b,h,t,0..P-1] (as written by
 * avq_attention with the same P and tile). Leaf ids outside [0, M0*(1+C))
 * and selected entries outside [0, M0) count only in the denominator; a
 * parent listed twice counts once. P == 0 gives 0 everywhere. A diagnostic
 * off the forward path: it costs an exact-attention pass (N^2 logits per
 * head, no values), fp32 logits from bf16 products, fp64 running sums.
 *
 * Supported: bf16, d in {64, 128}, tile 128 (fp32 inputs and tile 64:
 * AVQ_EUNSUPPORTED); a flat codebook (C == 0) takes P == 0 only.
 * Q, K: device [B,H,N,d] read only; assign: device [B,H,N] int32;
 * selected: device [B,H,ceil(N/tile),P] int32 (may be NULL when P == 0);
 * capture: device [B,H,N] float32, written. workspace: device,
 * >= avq_capture_workspace_bytes(s, P, tile) (the status word: a bounded
 * wait that ran out sets AVQ_ETIMEOUT).
 */
size_t avq_capture_workspace_bytes(const avq_shape* s, int P, int tile);
int avq_capture(const avq_shape* s, const void* Q, const void* K, const int32_t* assign,
                const int32_t* selected, int P, int tile, float scale, float* capture,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Query reordering along a Gilbert space-filling curve (paper §4.2,
 * "Per-query-tile amortization and adaptivity"; appendix "Spatial reordering
 * ablation", Table 8): tokens laid out on a rows x cols grid (token
 * t = r*cols + c) are reordered so that consecutive tokens are grid
 * neighbours and every run of T consecutive tokens (a query tile) covers a
 * compact 2-D region, for any grid size (the Gilbert curve generalises the
 * Hilbert curve to rectangles).
 *
 * avq_gilbert_order (host): order[i] = the token visited i-th, a permutation
 * of 0 .. rows*cols-1. order: host array of rows*cols int32, written.
 * Returns AVQ_OK or AVQ_EINVAL (rows or cols < 1, rows*cols >= 2^31, null).
 */
int avq_gilbert_order(int rows, int cols, int32_t* order);

/*
 * Row gather along the sequence (device): dst[b,h,i,:] = src[b,h,perm[i],:]
 * for i < s->N, with the row size of `s` (d elements of s->dtype). With
 * perm = a Gilbert order this reorders Q (or K, V) before the calls; with its
 * inverse it restores O afterwards. src, dst: device [B,H,N,d] (16-byte
 * aligned, not overlapping); perm: device, N int32, each in [0, N) (rows
 * outside are not read: dst row i is then zeroed). Returns AVQ_OK,
 * AVQ_EINVAL, AVQ_ECUDA. Does not synchronise.
 */
int avq_gather_rows(const avq_shape* s, const void* src, void* dst, const int32_t* perm, void* stream);

/*
 * Deeper codebook trees (paper §6 "Discussion and Conclusion": each further
 * level adds P*C codes to the attention cost per query and multiplies the
 * codebook's resolution by C; the pages propose it without testing it). The
 * two-level steps carried down every level of a depth-L tree:
 *
 *   codebook : [H, Mtot, d], Mtot = M0 (1 + C + ... + C^(L-1)); level l holds
 *              M0 C^l rows, stored level after level; node j of level l has
 *              the children j C + c (c < C) of level l + 1 (depth 2 is the
 *              avq_precompute layout). s->M0 = level-0 nodes, s->C = branching.
 *
 * avq_precompute_deep (paper §4.2 carried down): nearest level-0 node, then
 * level by level the nearest child of the current node replaces it only when
 * STRICTLY closer (ties to the lower index at every step); the descent stops
 * at the first level where no child is closer; assign = the last node's row.
 * Every node on a key's path counts the key and sums its V row (a node holds
 * all keys that reached it). Decisions are those of exact fp64 arithmetic
 * (distances summed in index order). counts/vsum are zeroed by the call.
 *
 * avq_attention_deep (paper §4.3 carried down): per query row one shift (the
 * largest level-0 logit of a non-empty node) and level-0 attention
 * A = exp(S - m), Zbar = sum A n, Xbar = sum A vsum; then for l = 0 .. L-2
 * the candidates (level 0: the M0 level-0 nodes; deeper: the children of
 * the nodes expanded at l - 1, in rank order) get the importance
 * sum_{i in tile} A_ic n_c / Zbar_i, with the Zbar so far; the P[l] largest
 * (ties to the lower row id) are expanded, and every child g of an expanded
 * node f adds (A_g - A_f) [vsum_g, n_g] to Xbar and Zbar. O = Xbar / Zbar.
 * P: host array of L-1 budgets, 0 <= P[l] <= (number of candidates at l) and
 * P[l] * C <= 128. selected: [B, H, ceil(N/tile), sum_l P[l]] int32, per
 * tile level 0's expanded row ids by rank, then level 1's, ...
 *
 * Supported: 2 <= L <= 4, 1 <= M0 <= 128, C >= 1, d in {64, 128}, fp32 or
 * bf16, tile in {64, 128}. Both calls run on CUDA cores (fp32 distances,
 * with exact fp64 ones wherever the fp32 error bound cannot decide; fp32
 * attention). The attention workspace (fp32 value means and the status
 * word) is avq_attention_deep_workspace_bytes(s, L) bytes, 256-byte
 * aligned. Errors: AVQ_EINVAL (arguments), AVQ_EUNSUPPORTED (sizes),
 * AVQ_EWORKSPACE, AVQ_ECUDA. Neither call synchronises.
 */
int avq_precompute_deep(const avq_shape* s, int L, const void* K, const void* V, const void* codebook,
                        int32_t* assign, int32_t* counts, float* vsum, void* stream);
size_t avq_attention_deep_workspace_bytes(const avq_shape* s, int L);
int avq_attention_deep(const avq_shape* s, int L, const int32_t* P, const void* Q, const void* codebook,
                       const int32_t* counts, const float* vsum, int tile, float scale, void* O,
                       int32_t* selected, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Blocking: waits for `stream`, then reads the status word that kernels of
 * earlier calls using `workspace` left there (AVQ_OK; AVQ_ETIMEOUT when a
 * bounded device-side wait ran out) and clears it.
 * Returns AVQ_ECUDA if the stream reports an error. A workspace must be
 * zero-filled before its first use.
 */
int avq_device_status(void* workspace, void* stream);

/*
 * Test hook for the failure path (no counterpart in the paper). The next
 * avq_attention call that runs the bf16 tensor-core tree kernel behaves as if
 * one of its bounded device-side waits had run out: the first wait of each
 * CTA's issuing thread (for its head's parent tables) gets a limit of zero.
 * Every CTA then stops
 * at once: the loads and contractions it has in flight complete, its tensor
 * memory is freed, and the call reports AVQ_ETIMEOUT through
 * avq_device_status (its outputs are not meaningful). Later calls are
 * unaffected. Returns AVQ_OK. Process-wide, consumed by one launch.
 */
int avq_test_fail_next_wait(void);

/* Human-readable name of a status code (static string). */
const char* avq_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int avq_version(void);

/*
 * Number of CUDA kernels this library has enqueued in this process so far
 * (all calls, all devices; host-side counter, thread-safe). Lets a caller
 * count the library's launches inside a timed region.
 */
uint64_t avq_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* AVQ_B200_H */
