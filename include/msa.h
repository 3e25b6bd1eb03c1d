/*
 * msa.h -- C ABI of libmsa_b200.so, the B200 (sm_100a) forward hot path of MiniMax Sparse Attention.
 *
 * Sources for what each call computes:
 *   [EXPL] "MiniMax Sparse Attention" explainer page: section 01 (causal GQA attention, G adjacent
 *          query heads share one KV head), section 02 (two-stage Index / Attn decomposition),
 *          Figure 1 (Index Branch: score, Block Max Pooling, Top-k per (query, GQA group) with the
 *          forced local block), section 04 (fixed budget k*B_k = 16*128), section 05-1 (exp-free
 *          Top-k), section 05-2 (KV-outer sparse attention, query concatenation, pre-scheduled
 *          chunking, two-stage forward with an LSE split-K combine, LSE emitted for the backward).
 *   [ABS]  The paper abstract ("MiniMax Sparse Attention", arXiv 2606.13392): Top-k per GQA
 *          group, exact block-sparse attention over the selected blocks, prefill and decoding.
 *   [BLOG] The "MiniMax M3" sparse-attention blog post, kernel paragraph: the attention kernels
 *          were tuned on FP8 tensor cores.
 *
 * Conventions shared by every entry point
 *   - bf16 tensors are passed as uint16_t bit patterns (msa_bf16).
 *   - Every tensor pointer is a DEVICE pointer into memory the caller allocated and owns; the
 *     library never allocates, frees or retains memory. Its only global state: the cached driver
 *     entry point used to encode TMA descriptors, the fixed scratch of msa_build_kv2q_static and
 *     the tracing hooks (msa_trace_set, msa_launch_count).
 *   - All work is enqueued asynchronously on `stream`. Exceptions: msa_get_device_error waits for
 *     the stream, and msa_sparse_prefill_varlen copies its host-side schedule from pageable
 *     memory (the copy may block the host until it is staged).
 *   - Arguments are validated on the host before anything is enqueued; a rejected call enqueues
 *     nothing and returns MSA_ERR_INVALID_ARG (bad pointer / shape / alignment),
 *     MSA_ERR_UNSUPPORTED (a valid shape this build has no kernel for) or MSA_ERR_WORKSPACE
 *     (workspace too small). Launch failures return MSA_ERR_CUDA.
 *   - Conditions only the device can see (a bounded wait that expired, a decode length outside
 *     [1, L_max]) are recorded in the device error word at the start of the workspace and read
 *     with msa_get_device_error(). No kernel traps.
 *   - Workspaces must be 256-byte aligned. Every entry point clears its own device error word.
 *   - Inputs must be finite. No C++ exception crosses this boundary.
 *
 * Supported shapes in this build: B_k = 128; 1 <= k <= 16; d_idx in {32, 64, 128};
 * d_h in {64, 128}; G = H_q / H_kv a power of two with G <= 128 (prefill) and G <= 16 (decode);
 * 1 <= N <= 2^21.
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

typedef uint16_t msa_bf16;
typedef struct CUstream_st* msa_stream_t; /* identical to cudaStream_t */

typedef enum {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARG = 1,
    MSA_ERR_UNSUPPORTED = 2,
    MSA_ERR_WORKSPACE = 3,
    MSA_ERR_CUDA = 4,
    MSA_ERR_TIMEOUT = 5,
    MSA_ERR_DEVICE_CHECK = 6
} msa_status;

/* Human-readable name of a status code (static storage). */
MSA_API const char* msa_status_string(msa_status status);

/* The CUDA call behind the calling thread's most recent MSA_ERR_CUDA, with its error name. */
MSA_API const char* msa_last_error_string(void);

/*
 * Reads the device error word of a workspace previously passed to an entry point (waits for
 * `stream` to finish). Returns MSA_OK, MSA_ERR_TIMEOUT (a bounded wait inside a kernel expired)
 * or MSA_ERR_DEVICE_CHECK (an input only the device can check was out of range), or
 * MSA_ERR_CUDA if the read itself failed.
 */
MSA_API msa_status msa_get_device_error(const void* workspace, msa_stream_t stream);

/*
 * Failure-path self-test (a diagnostic; the pages have no counterpart). Launches one thread that
 * waits, through the same bounded-wait routine every kernel of this library uses, on a barrier
 * phase that nothing completes. After `limit_cycles` SM clock cycles the wait gives up, records
 * MSA_ERR_TIMEOUT in the device error word at the start of `workspace` and the kernel returns:
 * msa_get_device_error() then reports MSA_ERR_TIMEOUT and the CUDA context stays usable.
 *   workspace       : >= msa_selftest_workspace_size() bytes, 256-byte aligned, caller-owned
 *   limit_cycles    : 1 .. 2,000,000,000 (about one second of SM clock at the upper end)
 * Returns MSA_ERR_INVALID_ARG / MSA_ERR_WORKSPACE before enqueueing anything, MSA_ERR_CUDA if the
 * launch failed, else MSA_OK (the timeout itself is read with msa_get_device_error).
 */
MSA_API size_t msa_selftest_workspace_size(void);
MSA_API msa_status msa_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int64_t limit_cycles,
                                             msa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Index Branch: fused index score + block max-pool + exp-free Top-k      [EXPL Fig. 1, 05-1]
 *
 * For every query row i and GQA group r:
 *   s_j      = q_idx[i, r, :] . k_idx[j, r, :]            (fp32 accumulation of bf16 products)
 *   S[i,r,b] = max over j in block b of s_j, for the fully visible blocks b < floor(i / B_k)
 *   set      = the k-1 blocks with the largest S (equal scores: lower block first) plus the local
 *              block floor(i / B_k); all visible blocks when floor(i / B_k) + 1 <= k.
 * No exp is evaluated (softmax preserves order). The pooled N x N/B_k score matrix is never
 * written to memory: scores go from tensor memory straight into per-row register Top-k lists.
 *
 *   q_idx, k_idx : [N, H_kv, d_idx] bf16, row-major, 16-byte aligned
 *   block_idx    : [H_kv, N, k] int32 out; each row ascending, padded with -1
 *   workspace    : >= msa_index_topk_workspace_size(...) bytes (error word + scheduler state)
 * Index inputs whose scores are exact in fp32 (e.g. small integers) give selections identical
 * to an exact-arithmetic reference.
 * ------------------------------------------------------------------------------------------ */
MSA_API size_t msa_index_topk_workspace_size(int64_t N, int H_kv, int d_idx, int B_k, int k);

MSA_API msa_status msa_index_topk(const msa_bf16* q_idx, const msa_bf16* k_idx, int64_t N, int H_kv, int d_idx, int B_k,
                          int k, int32_t* block_idx, void* workspace, size_t workspace_bytes, msa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * KV -> Q inversion with pre-scheduled chunking                                  [EXPL 05-2]
 *
 * Turns the per-query selections into per-KV-block lists of the query rows that selected the
 * block ("KV-outer": each K/V block gathers its queries), plus a work list for the attention.
 *
 * The result lives in ONE caller-allocated device buffer `kv2q` of layout.total_bytes bytes,
 * described by a host-side msa_kv2q_layout filled by msa_kv2q_layout_get(). Arrays in it:
 *   offsets      int32 [H_kv][nb + 1]  CSR row pointers per group; offsets[r][0] = 0
 *   entries      int32 [H_kv][N * k]   list of block b of group r = entries[r][offsets[r][b] ..
 *                                      offsets[r][b+1]), rows ascending, each entry i*k + slot
 *                                      (slot = rank of b in row i's ascending set)
 *   items        msa_work_item [max_items]  ordered window-major: all items whose rows lie in
 *                                      query window w (rows [w*window, (w+1)*window)) precede
 *                                      those of window w+1; inside a window, by (r, b). An item
 *                                      covers at most `chunk` consecutive entries of one list.
 *   window_items int32 [n_windows + 1] first item of each window; the last value is the count
 *   (plus internal per-(r, b, window) counts used while building)
 * window = 0 / chunk = 0 select the defaults: windows of N / 128 rows rounded up to a power of two
 * within [2048, 16384] (2048 up to N = 256K; longer sequences get longer windows so that each
 * (window, block) item keeps its 128-row tiles nearly full), items of at most 512 entries.
 * ------------------------------------------------------------------------------------------ */
typedef struct {
    int32_t r;     /* GQA group */
    int32_t b;     /* KV block */
    int32_t start; /* first entry, index into entries[r] */
    int32_t len;   /* number of entries */
} msa_work_item;

typedef struct {
    int64_t N;
    int32_t H_kv, B_k, k, nb;
    int32_t window, chunk, n_windows;
    int64_t max_items;
    size_t offsets, entries, items, window_items, counts, bases; /* byte offsets into the buffer */
    size_t total_bytes;
} msa_kv2q_layout;

MSA_API msa_status msa_kv2q_layout_get(int64_t N, int H_kv, int B_k, int k, int window, int chunk, msa_kv2q_layout* layout);

MSA_API size_t msa_build_kv2q_workspace_size(const msa_kv2q_layout* layout);

/*   block_idx : [H_kv, N, k] int32 as written by msa_index_topk (ascending, -1 padded)
 *   layout    : host struct from msa_kv2q_layout_get with the same N, H_kv, B_k, k
 *   kv2q      : device buffer of layout->total_bytes bytes, filled by this call */
MSA_API msa_status msa_build_kv2q(const int32_t* block_idx, const msa_kv2q_layout* layout, void* kv2q, void* workspace,
                          size_t workspace_bytes, msa_stream_t stream);

/*
 * msa_build_kv2q_static: the same inversion as msa_build_kv2q, for callers that cannot allocate
 * device memory. The pages have no counterpart; this is an interface variant, not a step of the
 * method. Typical such callers are plug-ins handed only their input and output buffers by a host
 * framework that owns every device allocation, and latency-critical loops where a cudaMalloc or
 * cudaFree would synchronise the device.
 *   - No workspace argument and no allocation: the scratch (device error word + scan partials)
 *     is a fixed 1 MiB array of this library (a file-scope __device__ array), held by every GPU
 *     that loads the library until the process exits. The caller still passes block_idx, the
 *     layout and the kv2q output buffer, exactly as for msa_build_kv2q.
 *   - The first call on a device looks up the array's device address on that device (it must be
 *     the current device); make that first call before any stream capture. On every call
 *     `stream` must belong to the current device (else MSA_ERR_INVALID_ARG): the array's address
 *     differs between GPUs.
 *   - The layout is validated exactly as msa_build_kv2q validates it (every field, including nb
 *     and n_windows, must be what msa_kv2q_layout_get returns); a mismatch is MSA_ERR_INVALID_ARG.
 *   - Layouts whose scratch would exceed 1 MiB are rejected with MSA_ERR_WORKSPACE (every shape
 *     this build supports fits: the scan needs one int32 per 1024 (group, block, window) counters).
 *   - All calls share the one array: calls whose work overlaps on the GPU (other streams, other
 *     threads) race on it. The error word is cleared at the start of every call; the variant
 *     does not expose it, so out-of-range block ids are skipped without a report.
 */
MSA_API msa_status msa_build_kv2q_static(const int32_t* block_idx, const msa_kv2q_layout* layout, void* kv2q,
                                         msa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Main Branch: exact block-sparse causal attention, KV-outer, two-stage      [EXPL 05-2, ABS]
 *
 * For row i, head h (group r = floor(h / G)) and T = {j <= i : block(j) in set(i, r)}:
 *   out[i, h] = sum_{j in T} softmax_T(q[i,h] . k[j,r] / sqrt(d_h)) v[j, r]
 *   lse[i, h] = log sum_{j in T} exp(q[i,h] . k[j,r] / sqrt(d_h))   (natural log, scaled logits)
 * Stage 1 walks the work list: each item stages its K/V block once and gathers 128/G query
 * rows x G heads per 128-row tensor-core tile, writing a partial (normalised output, lse) per
 * (row, head, slot). Stage 2 merges the <= k partials of each (row, head) through their lse.
 *
 *   q        : [N, H_q, d_h] bf16;   k, v : [N, H_kv, d_h] bf16  (16-byte aligned)
 *   block_idx: [H_kv, N, k] int32 (msa_index_topk output)
 *   layout, kv2q : a built inversion, or both NULL to build it inside the workspace
 *   out      : [N, H_q, d_h] bf16 out;  lse : [N, H_q] fp32 out, or NULL
 *   workspace: >= msa_sparse_prefill_workspace_size(..., max_rows_per_pass, internal_kv2q).
 *              Partials need about H_q * k * (2*d_h + 4) bytes per query row; when the workspace
 *              holds fewer rows than N the call processes the query windows in passes.
 * ------------------------------------------------------------------------------------------ */
MSA_API size_t msa_sparse_prefill_workspace_size(int64_t N, int H_q, int H_kv, int d_h, int B_k, int k,
                                         int64_t max_rows_per_pass, int internal_kv2q);

MSA_API msa_status msa_sparse_prefill(const msa_bf16* q, const msa_bf16* k, const msa_bf16* v, int64_t N, int H_q, int H_kv,
                              int d_h, int B_k, int kk, const int32_t* block_idx, const msa_kv2q_layout* layout,
                              const void* kv2q, msa_bf16* out, float* lse, void* workspace, size_t workspace_bytes,
                              msa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * FP8 main branch                               [BLOG: kernel paragraph, FP8 tensor cores]
 *
 * The page names FP8 tensor cores for the attention kernels and gives no quantisation; reading:
 * q, k and v are quantised row by row, one scale per (token, head) row, to OCP E4M3 (bias 7,
 * subnormals, largest finite 448, no infinities): scale = amax / 448 (1 for an all-zero row),
 * code = nearest E4M3 value of x / scale (ties to the even code, |x / scale| >= 448 saturates).
 * The main branch is then the exact attention of msa_sparse_prefill on the dequantised values
 * code * scale.
 *
 * msa_quantize_e4m3: x [N, H, d] bf16 (d in {64, 128}) ->
 *   codes   : [N, H, d] uint8 E4M3 codes (the quotient x / scale is formed in fp64, so codes are
 *             bit-identical to the definition above)
 *   scales  : [H, S] fp32, S = N rounded up to a multiple of 128 (head-major; tokens N..S-1 get 1)
 *   rscales : [H, S] fp32 = 1 / scales, or NULL
 *   blkmax  : [H, S / 128] fp32 = largest scale of each 128-token block, or NULL (cleared here)
 * All device pointers 16-byte aligned (blkmax 4). Asynchronous on `stream`, no workspace.
 *
 * msa_sparse_prefill_fp8: the main branch on E4M3 inputs (d_h = 128, G <= 16): q8, qs from
 * msa_quantize_e4m3 of q; k8, ks of k; v8, vs, rvs, vblkmax of v (all three outputs). The S = QK^T
 * and PV products run on the FP8 tensor cores (tcgen05 kind::f8f6f4) with fp32 accumulation; the
 * k scales enter the logits per key, the q scale per row; the attention weights P are scaled by
 * the key's v scale and 448 / (the block's largest v scale) and rounded to E4M3 for the PV product,
 * and each partial output is normalised by the sum of the weights those codes stand for (so it is
 * an exact weighted average of V rows); the lse uses the unrounded weights. Arguments, layout,
 * workspace (msa_sparse_prefill_workspace_size) and outputs as for msa_sparse_prefill.
 * ------------------------------------------------------------------------------------------ */
MSA_API msa_status msa_quantize_e4m3(const msa_bf16* x, int64_t N, int H, int d, uint8_t* codes, float* scales,
                                     float* rscales, float* blkmax, msa_stream_t stream);

MSA_API msa_status msa_sparse_prefill_fp8(const uint8_t* q8, const float* qs, const uint8_t* k8, const float* ks,
                                          const uint8_t* v8, const float* vs, const float* rvs, const float* vblkmax,
                                          int64_t N, int H_q, int H_kv, int d_h, int B_k, int k,
                                          const int32_t* block_idx, const msa_kv2q_layout* layout, const void* kv2q,
                                          msa_bf16* out, float* lse, void* workspace, size_t workspace_bytes,
                                          msa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Backward: main-branch gradients (selections fixed) and the index-branch KL signal [EXPL 03, 05]
 *
 * The Top-k selection is not differentiable, so the loss reaches q, k and v only through the
 * exact attention of msa_sparse_prefill over each row's token set T. With p_j the attention
 * weights of (i, h) (recomputed from q, k and the forward's lse), D = dout[i,h] . out[i,h] and
 * ds_j = p_j (dout[i,h] . v[j,r] - D):
 *   dq[i, h] = sum_{j in T} ds_j k[j, r] / sqrt(d_h)
 *   dk[j, r] = sum over (i, h in group r) with j in T(i, r) of ds_j q[i, h] / sqrt(d_h)
 *   dv[j, r] = sum over the same (i, h) of p_j dout[i, h]
 * KV-outer over the inversion's work items: each item stages its K/V block once, walks its rows
 * in 16-row tiles and keeps the block's dK and dV in registers; dq and the item's dk, dv are added
 * to fp32 accumulators in the workspace and rounded to bf16 at the end.
 *
 * Optional, in the same pass (q_idx != NULL): the index branch's KL alignment [EXPL 03 "KL Loss"].
 * Over T(i, r) the student is P_idx = softmax(q_idx[i,r] . k_idx[j,r]) (unscaled index scores), the
 * teacher P = the mean of the group's G attention weights above; KL(i, r) = sum_j P_j log(P_j /
 * P_idx_j), teacher stop-gradient, so with w = kl_weight (1 / (N * H_kv) for the mean):
 *   dq_idx[i, r] = w sum_{j in T} (P_idx_j - P_j) k_idx[j, r]
 *   dk_idx[j, r] = w sum over rows i with j in T(i, r) of (P_idx_j - P_j) q_idx[i, r]
 *   kl[i, r]     = KL(i, r) (unweighted), when kl != NULL
 *
 *   q, out, dout : [N, H_q, d_h] bf16 (out: the forward's output, dout: upstream gradient)
 *   k, v     : [N, H_kv, d_h] bf16;  lse : [N, H_q] fp32 (the forward's lse, required)
 *   block_idx: [H_kv, N, k] int32 (the forward's selections); may be NULL when layout/kv2q are given
 *   layout, kv2q : the forward's inversion, or both NULL to build it inside the workspace
 *   dq : [N, H_q, d_h] bf16 out;  dk, dv : [N, H_kv, d_h] bf16 out
 *   q_idx, k_idx : [N, H_kv, d_idx] bf16 (the index branch's inputs), or q_idx = NULL to skip the KL
 *              part (then k_idx, d_idx, kl_weight, dq_idx, dk_idx, kl are ignored); needs block_idx
 *   dq_idx, dk_idx : [N, H_kv, d_idx] bf16 out;  kl : [N, H_kv] fp32 out, or NULL
 *   workspace: >= msa_sparse_backward_workspace_size(..., d_idx or 0 without KL, internal_kv2q) bytes,
 *              256-byte aligned (fp32 accumulators: 4 * N * d_h * (H_q + 2 * H_kv) bytes plus
 *              4 * N * H_q, and with KL 4 * N * H_kv * (2 * d_idx + 1))
 * All tensor pointers 16-byte aligned (lse 4). Supported: B_k = 128, k <= 16, d_h in {64, 128},
 * G = H_q / H_kv in {1, 2, 4, 8, 16}, d_idx in {32, 64} for the KL part. Errors:
 * MSA_ERR_INVALID_ARG, MSA_ERR_UNSUPPORTED, MSA_ERR_WORKSPACE, MSA_ERR_CUDA; entries outside
 * [0, N) are skipped and recorded in the device error word (MSA_ERR_DEVICE_CHECK).
 * msa_sparse_backward_workspace_size returns 0 for arguments the call would reject.
 * ------------------------------------------------------------------------------------------ */
MSA_API size_t msa_sparse_backward_workspace_size(int64_t N, int H_q, int H_kv, int d_h, int B_k, int k,
                                                  int d_idx, int internal_kv2q);

MSA_API msa_status msa_sparse_backward(const msa_bf16* q, const msa_bf16* k, const msa_bf16* v, const msa_bf16* out,
                                       const float* lse, const msa_bf16* dout, int64_t N, int H_q, int H_kv, int d_h,
                                       int B_k, int kk, const int32_t* block_idx, const msa_kv2q_layout* layout,
                                       const void* kv2q, msa_bf16* dq, msa_bf16* dk, msa_bf16* dv,
                                       const msa_bf16* q_idx, const msa_bf16* k_idx, int d_idx, float kl_weight,
                                       msa_bf16* dq_idx, msa_bf16* dk_idx, float* kl, void* workspace,
                                       size_t workspace_bytes, msa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Packed-batch (varlen) prefill: the whole forward for B independent sequences  [EXPL 05, ABS]
 *
 * Sequence s has query rows cu_seqlens[s] .. cu_seqlens[s+1]-1 of the packed query tensors and key
 * rows cu_seqlens_k[s] .. cu_seqlens_k[s+1]-1 of the packed key tensors. Each sequence is its own
 * causal problem with the definitions of msa_index_topk and msa_sparse_prefill applied to its
 * tokens alone: its blocks are numbered from 0 at its first token, rows never see another
 * sequence's tokens. When a sequence has more keys than queries (chunked prefill continuing from a
 * KV cache: the keys hold the cached prefix followed by the chunk), its queries are its LAST
 * positions: query row r of the sequence sits at position (len_k - len_q) + r, and the prefix
 * length len_k - len_q must be a whole number of blocks. One call runs the index branch, the
 * inversion (keyed on the blocks of all sequences), the attention and the combine.
 *
 *   q, q_idx : [T, H_q, d_h], [T, H_kv, d_idx] bf16, T = cu_seqlens[B] query rows
 *   k, v, k_idx : [Tk, H_kv, d_h], [Tk, H_kv, d_idx] bf16, Tk = cu_seqlens_k[B] key rows
 *              (all 16-byte aligned)
 *   cu_seqlens, cu_seqlens_k: HOST arrays [B+1] starting at 0, non-decreasing (empty sequences
 *              allowed); cu_seqlens_k may be NULL (keys packed like the queries, no prefixes);
 *              read before the call returns (they size the schedule, which is copied to the device)
 *   block_idx: [H_kv, T, k] int32 out: each row's selection as block indices local to its
 *              sequence, ascending, -1 padded (as msa_index_topk for that sequence alone)
 *   out      : [T, H_q, d_h] bf16 out;  lse : [T, H_q] fp32 out, or NULL
 *   workspace: >= msa_sparse_prefill_varlen_workspace_size(cu_seqlens, B, ..., max_rows_per_pass)
 *              bytes, 256-byte aligned, caller-owned; smaller workspaces run the attention in passes
 *              of whole query windows, down to one window
 * Errors: MSA_ERR_INVALID_ARG (NULL/misaligned pointers, bad cu_seqlens, fewer keys than queries
 * in a sequence), MSA_ERR_UNSUPPORTED (shapes outside this build, a prefix that is not a whole
 * number of blocks), MSA_ERR_WORKSPACE, MSA_ERR_CUDA; device checks as msa_sparse_prefill.
 * msa_sparse_prefill_varlen_workspace_size returns 0 for arguments the call would reject.
 * ------------------------------------------------------------------------------------------ */
MSA_API size_t msa_sparse_prefill_varlen_workspace_size(const int32_t* cu_seqlens, const int32_t* cu_seqlens_k, int B,
                                                        int H_q, int H_kv, int d_h, int B_k, int k,
                                                        int64_t max_rows_per_pass);

MSA_API msa_status msa_sparse_prefill_varlen(const msa_bf16* q, const msa_bf16* k, const msa_bf16* v,
                                             const msa_bf16* q_idx, const msa_bf16* k_idx, const int32_t* cu_seqlens,
                                             const int32_t* cu_seqlens_k, int B, int H_q, int H_kv, int d_h, int d_idx,
                                             int B_k, int kk,
                                             int32_t* block_idx, msa_bf16* out, float* lse, void* workspace,
                                             size_t workspace_bytes, msa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Decode: one query token per sequence against a KV cache                  [ABS, EXPL Fig. 4]
 *
 * Sequence beta holds lens[beta] cached tokens (the current token included) and its query sits
 * at position i = lens[beta] - 1; selection and attention are those of prefill row i of that
 * sequence. The index scores stream over the k_idx cache split across CTAs, per-lane register
 * Top-k lists are merged with warp shuffles, then split attention over the k selected blocks is
 * merged through the lse like prefill.
 *
 *   q       : [B, H_q, d_h] bf16;  q_idx : [B, H_kv, d_idx] bf16
 *   k_cache, v_cache : [B, L_max, H_kv, d_h] bf16;  k_idx_cache : [B, L_max, H_kv, d_idx] bf16
 *   lens    : [B] int32 device array, 1 <= lens[beta] <= L_max (checked on the device; a bad
 *             length sets MSA_ERR_DEVICE_CHECK and that sequence's output is left unwritten)
 *   out     : [B, H_q, d_h] bf16 out;  lse : [B, H_q] fp32 out or NULL
 *   block_idx_out : [B, H_kv, k] int32 out or NULL (the selections)
 * ------------------------------------------------------------------------------------------ */
MSA_API size_t msa_sparse_decode_workspace_size(int B, int64_t L_max, int H_q, int H_kv, int d_h, int d_idx, int B_k, int k);

MSA_API msa_status msa_sparse_decode(const msa_bf16* q, const msa_bf16* q_idx, const msa_bf16* k_cache,
                             const msa_bf16* v_cache, const msa_bf16* k_idx_cache, const int32_t* lens, int B,
                             int64_t L_max, int H_q, int H_kv, int d_h, int d_idx, int B_k, int k, msa_bf16* out,
                             float* lse, int32_t* block_idx_out, void* workspace, size_t workspace_bytes,
                             msa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Tracing (measurement support; no counterpart on the pages)
 *
 * msa_trace_set() installs a caller-owned record: while installed, every entry point records
 * events[2j] / events[2j+1] (caller-created cudaEvent_t handles) on its stream immediately
 * before / after its j-th traced kernel and stores that kernel's id in kernel_ids[j]; `count`
 * advances by 2 per traced kernel and recording stops silently at `capacity`. NULL uninstalls.
 * Process-wide and not thread-safe: one tracing caller at a time. msa_launch_count() returns the
 * number of kernels this library has launched in the process (for launch accounting).
 * ------------------------------------------------------------------------------------------ */
typedef enum {
    MSA_KERNEL_INDEX_TOPK = 1, /* fused index score + max-pool + Top-k                         */
    MSA_KERNEL_KV2Q = 2,       /* whole KV->Q inversion (count, scans, scatter, work list)      */
    MSA_KERNEL_ATTN = 3,       /* KV-outer attention, stage 1 (one per pass)                    */
    MSA_KERNEL_COMBINE = 4,    /* LSE combine, stage 2 (one per pass)                           */
    MSA_KERNEL_DEC_POOL = 5,   /* decode index scores + max-pool                                */
    MSA_KERNEL_DEC_TOPK = 6,   /* decode Top-k warp merge                                       */
    MSA_KERNEL_DEC_ATTN = 7,   /* decode split attention                                        */
    MSA_KERNEL_DEC_COMBINE = 8, /* decode LSE combine                                           */
    MSA_KERNEL_BWD_PREP = 9,    /* backward: rowsum(dout * out)                                 */
    MSA_KERNEL_BWD_ATTN = 10,   /* backward: KV-outer gradients                                 */
    MSA_KERNEL_BWD_CONVERT = 11, /* backward: fp32 accumulators to bf16                         */
    MSA_KERNEL_QUANT = 12       /* E4M3 quantisation of one tensor                               */
} msa_kernel_id;

typedef struct {
    void** events;   /* cudaEvent_t handles, two per traced kernel */
    int capacity;    /* number of handles in events */
    int count;       /* handles used so far (written by the library) */
    int* kernel_ids; /* [capacity / 2] msa_kernel_id of each traced kernel (written) */
} msa_trace;

MSA_API void msa_trace_set(msa_trace* trace);

MSA_API uint64_t msa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H */
