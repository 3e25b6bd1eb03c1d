// msa_api.cu -- the C ABI of libmsa_b200.so (declared in include/msa.h): host-side validation,
// workspace carving, TMA descriptor encoding and kernel launches. No allocation, no host sync.
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <algorithm>
#include <vector>

#include "backward.cuh"
#include "common.cuh"
#include "sm100.cuh"

using namespace msa;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D tensor [n2][n1][n0] (row-major) of bf16 (eb = 2) or 8-bit codes (eb = 1), box {b0, b1, b2}.
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t n0, uint64_t n1, uint64_t n2, uint32_t b0, uint32_t b1,
                 uint32_t b2, CUtensorMapSwizzle sw, int eb = 2)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {n0, n1, n2};
    const cuuint64_t strides[2] = {n0 * eb, n0 * n1 * eb};
    const cuuint32_t box[3] = {b0, b1, b2};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, eb == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base),
              dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Query map of the attention's row gather. G >= 8: one box per position holds its G heads x d_h
// columns: a 5-D view of q[N][H_q][d_h] with dims (64 columns, 8 heads, 64-column chunk, head group
// of 8, position), so the box lands in shared memory as [head group][chunk][8 heads][128 B] and the
// tile's 8-row groups are a uniform 1024 * d_h / 64 bytes apart. G < 8: one 3-D box of G heads x 64
// columns per 64-column chunk.
bool make_qmap(CUtensorMap* m, const void* q, int d_h, int H_q, int64_t N, int G, int eb = 2)
{
    const uint32_t ce = 128 / eb; // elements per 128-byte chunk
    if (G < 8) return make_map_3d(m, q, d_h, H_q, N, ce, G, 1, CU_TENSOR_MAP_SWIZZLE_128B, eb);
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t nkc = (cuuint64_t)d_h / ce;
    const cuuint64_t row = (cuuint64_t)d_h * eb;
    const cuuint64_t dims[5] = {ce, 8, nkc, (cuuint64_t)H_q / 8, (cuuint64_t)N};
    const cuuint64_t strides[4] = {row, 128, 8 * row, (cuuint64_t)H_q * row};
    const cuuint32_t box[5] = {ce, 8, (cuuint32_t)nkc, (cuuint32_t)(G / 8), 1};
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, eb == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(q),
              dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

bool injected(const char* name)
{
    const char* v = getenv("MSA_FAULT_INJECT");
    return v && strcmp(v, name) == 0;
}

constexpr size_t kErrBytes = 256;
constexpr int kDefaultWindow = 2048;
constexpr int kDefaultChunk = 512;

// Default query window: N / 128 rounded up to a power of two within [2048, 16384] for one sequence
// (nb = ceil(N / 128)), 2048 for a packed batch. A window's rows select about W * (k - 1) / (visible
// blocks) rows per (window, block) item, ~30 at mid-sequence with W = N / 128, so the 128-row tiles of
// an item stay nearly full on long sequences, while short ones keep small windows whose gathered
// query rows stay in L2.
int default_window(int64_t N, int64_t nb)
{
    if (nb != (N + kBk - 1) / kBk) return kDefaultWindow; // packed batch of sequences
    int w = kDefaultWindow;
    while (w < 16384 && (int64_t)w < N / kBk) w *= 2;
    return w;
}

size_t kv2q_internal_tmp(const msa_kv2q_layout& L)
{
    return kv2q_scan_tmp_bytes((int64_t)L.H_kv * L.nb * L.n_windows, L.H_kv);
}

thread_local char g_last_error[256] = "no error";

// Records the failing CUDA call of the last MSA_ERR_CUDA (per thread) for msa_last_error_string().
msa_status cuda_status(cudaError_t e, const char* site)
{
    if (e == cudaSuccess) return MSA_OK;
    snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", site, cudaGetErrorName(e), cudaGetErrorString(e));
    return MSA_ERR_CUDA;
}

msa_trace* g_trace = nullptr;
std::atomic<uint64_t> g_launches{0};

} // namespace

namespace msa {

// A record that fails (e.g. a handle that is not a live event) ends tracing for this record and
// clears the error, so that it is never mistaken for a launch failure.
static bool trace_record(msa_trace* t, int slot, cudaStream_t s)
{
    if (t->events[slot] && cudaEventRecord((cudaEvent_t)t->events[slot], s) == cudaSuccess) return true;
    cudaGetLastError();
    t->capacity = t->count;
    return false;
}

void trace_begin(cudaStream_t s)
{
    msa_trace* t = g_trace;
    if (t && t->count + 2 <= t->capacity) trace_record(t, t->count, s);
}

void trace_end(cudaStream_t s, int kernel_id)
{
    msa_trace* t = g_trace;
    if (t && t->count + 2 <= t->capacity && trace_record(t, t->count + 1, s)) {
        t->kernel_ids[t->count / 2] = kernel_id;
        t->count += 2;
    }
}

void note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

} // namespace msa

extern "C" {

void msa_trace_set(msa_trace* trace) { g_trace = trace; }

const char* msa_last_error_string(void) { return g_last_error; }

uint64_t msa_launch_count(void) { return g_launches.load(); }

const char* msa_status_string(msa_status s)
{
    switch (s) {
    case MSA_OK: return "MSA_OK";
    case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG";
    case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED";
    case MSA_ERR_WORKSPACE: return "MSA_ERR_WORKSPACE";
    case MSA_ERR_CUDA: return "MSA_ERR_CUDA";
    case MSA_ERR_TIMEOUT: return "MSA_ERR_TIMEOUT";
    case MSA_ERR_DEVICE_CHECK: return "MSA_ERR_DEVICE_CHECK";
    }
    return "MSA_ERR_UNKNOWN";
}

msa_status msa_get_device_error(const void* workspace, msa_stream_t stream)
{
    if (!workspace) return MSA_ERR_INVALID_ARG;
    int h[2] = {0, 0};
    if (cudaMemcpyAsync(h, workspace, sizeof h, cudaMemcpyDeviceToHost, (cudaStream_t)stream) != cudaSuccess ||
        cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
        return MSA_ERR_CUDA;
    return (msa_status)h[0];
}

// ------------------------------------------------------------------------------------ self-test
size_t msa_selftest_workspace_size(void) { return kErrBytes; }

msa_status msa_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int64_t limit_cycles,
                                     msa_stream_t stream)
{
    if (!workspace || !aligned(workspace, 256) || limit_cycles < 1 || limit_cycles > 2000000000LL)
        return MSA_ERR_INVALID_ARG;
    if (workspace_bytes < kErrBytes) return MSA_ERR_WORKSPACE;
    if (injected("msa_selftest_wait_timeout")) return MSA_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    if (msa_status st0 = cuda_status(cudaMemsetAsync(workspace, 0, kErrBytes, s), "clearing the error word")) return st0;
    return cuda_status(launch_selftest_wait((int*)workspace, (long long)limit_cycles, s), "self-test launch");
}

// ------------------------------------------------------------------------------------ index_topk
size_t msa_index_topk_workspace_size(int64_t, int, int, int, int) { return kErrBytes; }

msa_status msa_index_topk(const msa_bf16* q_idx, const msa_bf16* k_idx, int64_t N, int H_kv, int d_idx, int B_k,
                          int k, int32_t* block_idx, void* workspace, size_t workspace_bytes, msa_stream_t stream)
{
    if (!q_idx || !k_idx || !block_idx || !workspace || N < 1 || H_kv < 1 || k < 1 || d_idx < 1 || B_k < 1)
        return MSA_ERR_INVALID_ARG;
    if (!aligned(q_idx, 16) || !aligned(k_idx, 16) || !aligned(block_idx, 4) || !aligned(workspace, 256))
        return MSA_ERR_INVALID_ARG;
    if (B_k != kBk || k > kMaxK || !(d_idx == 32 || d_idx == 64 || d_idx == 128) || N > kMaxN || H_kv > 65535)
        return MSA_ERR_UNSUPPORTED;
    if (workspace_bytes < kErrBytes) return MSA_ERR_WORKSPACE;
    if (injected("msa_index_topk")) return MSA_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    CUtensorMap qmap, kmap;
    const uint32_t box0 = d_idx < 64 ? (uint32_t)d_idx : 64u;
    const CUtensorMapSwizzle sw = d_idx == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_map_3d(&qmap, q_idx, d_idx, H_kv, N, box0, 1, kBk, sw) ||
        !make_map_3d(&kmap, k_idx, d_idx, H_kv, N, box0, 1, kBk, sw))
        return MSA_ERR_INVALID_ARG;
    if (msa_status st0 = cuda_status(cudaMemsetAsync(workspace, 0, kErrBytes, s), "clearing the error word")) return st0;
    IndexTopkArgs a{q_idx, k_idx, N, H_kv, d_idx, k, block_idx, (int*)workspace};
    trace_begin(s);
    const cudaError_t e = launch_index_topk(a, qmap, kmap, s);
    trace_end(s, MSA_KERNEL_INDEX_TOPK);
    return cuda_status(e, "index_topk launch");
}

// ------------------------------------------------------------------------------------ kv2q
} // extern "C"

// Layout of an inversion over N rows whose selections name nb distinct blocks (nb = ceil(N / B_k)
// for one sequence; the sum of the sequences' block counts for a packed batch).
static msa_status layout_fill(int64_t N, int H_kv, int B_k, int k, int64_t nb, int window, int chunk,
                              msa_kv2q_layout* L)
{
    if (!L || N < 1 || H_kv < 1 || B_k < 1 || k < 1 || window < 0 || chunk < 0 || nb < 1) return MSA_ERR_INVALID_ARG;
    if (B_k != kBk || k > kMaxK || N > kMaxN || nb > (int64_t)kMaxN) return MSA_ERR_UNSUPPORTED;
    if (window == 0) window = default_window(N, nb);
    if (chunk == 0) chunk = kDefaultChunk < window ? kDefaultChunk : window;
    if (window % kBk != 0 || chunk > window) return MSA_ERR_INVALID_ARG;
    memset(L, 0, sizeof *L);
    L->N = N;
    L->H_kv = H_kv;
    L->B_k = B_k;
    L->k = k;
    L->nb = (int32_t)nb;
    L->window = window;
    L->chunk = chunk;
    L->n_windows = (int32_t)((N + window - 1) / window);
    int64_t max_items = 0;
    for (int64_t w = 0; w < L->n_windows; ++w) {
        const int64_t lo = w * window, hi = (w + 1) * window < N ? (w + 1) * window : N;
        const int64_t vis_one = (hi - 1) / B_k + 1; // blocks visible to the window's rows (one sequence)
        const int64_t vis = vis_one < nb ? vis_one : nb;
        max_items += (int64_t)H_kv * (vis + ((hi - lo) * k + chunk - 1) / chunk);
    }
    L->max_items = max_items;
    const int64_t n = (int64_t)H_kv * L->nb * L->n_windows;
    size_t off = 0;
    L->offsets = off;
    off = align_up(off + (size_t)H_kv * (L->nb + 1) * 4, 256);
    L->entries = off;
    off = align_up(off + (size_t)H_kv * N * k * 4, 256);
    L->items = off;
    off = align_up(off + (size_t)max_items * sizeof(msa_work_item), 256);
    L->window_items = off;
    off = align_up(off + (size_t)(L->n_windows + 1) * 4, 256);
    L->counts = off;
    off = align_up(off + (size_t)2 * n * 4, 256);
    L->bases = off;
    off = align_up(off + (size_t)n * 4, 256);
    L->total_bytes = off;
    return MSA_OK;
}

extern "C" {

msa_status msa_kv2q_layout_get(int64_t N, int H_kv, int B_k, int k, int window, int chunk, msa_kv2q_layout* L)
{
    if (!L || N < 1 || B_k < 1) return MSA_ERR_INVALID_ARG;
    return layout_fill(N, H_kv, B_k, k, (N + B_k - 1) / B_k, window, chunk, L);
}

size_t msa_build_kv2q_workspace_size(const msa_kv2q_layout* L)
{
    return L ? kErrBytes + kv2q_internal_tmp(*L) : 0;
}

static msa_status build_kv2q_impl(const int32_t* block_idx, const msa_kv2q_layout* L, void* kv2q, int* err,
                                  void* tmp, cudaStream_t s, const int32_t* row_start = nullptr,
                                  const int32_t* row_gb0 = nullptr)
{
    uint8_t* base = (uint8_t*)kv2q;
    Kv2qArgs a;
    a.block_idx = block_idx;
    a.N = L->N;
    a.H_kv = L->H_kv;
    a.k = L->k;
    a.nb = L->nb;
    a.window = L->window;
    a.chunk = L->chunk;
    a.n_windows = L->n_windows;
    a.offsets = (int32_t*)(base + L->offsets);
    a.entries = (int32_t*)(base + L->entries);
    a.items = (msa_work_item*)(base + L->items);
    a.window_items = (int32_t*)(base + L->window_items);
    a.counts = (int32_t*)(base + L->counts);
    a.bases = (int32_t*)(base + L->bases);
    a.max_items = L->max_items;
    a.scan_tmp = (int32_t*)tmp;
    a.err = err;
    a.row_start = row_start;
    a.row_gb0 = row_gb0;
    trace_begin(s);
    const cudaError_t e = launch_kv2q(a, s);
    trace_end(s, MSA_KERNEL_KV2Q);
    return cuda_status(e, "kv2q launch");
}

static bool layout_ok(const msa_kv2q_layout* L)
{
    msa_kv2q_layout ref;
    if (msa_kv2q_layout_get(L->N, L->H_kv, L->B_k, L->k, L->window, L->chunk, &ref) != MSA_OK) return false;
    return ref.nb == L->nb && ref.n_windows == L->n_windows && ref.max_items == L->max_items &&
           ref.offsets == L->offsets && ref.entries == L->entries && ref.items == L->items &&
           ref.window_items == L->window_items && ref.counts == L->counts && ref.bases == L->bases &&
           ref.total_bytes == L->total_bytes;
}

msa_status msa_build_kv2q(const int32_t* block_idx, const msa_kv2q_layout* L, void* kv2q, void* workspace,
                          size_t workspace_bytes, msa_stream_t stream)
{
    if (!block_idx || !L || !kv2q || !workspace) return MSA_ERR_INVALID_ARG;
    if (!layout_ok(L) || !aligned(kv2q, 256) || !aligned(workspace, 256) || !aligned(block_idx, 4))
        return MSA_ERR_INVALID_ARG;
    if (workspace_bytes < msa_build_kv2q_workspace_size(L)) return MSA_ERR_WORKSPACE;
    if (injected("msa_build_kv2q")) return MSA_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    if (msa_status st0 = cuda_status(cudaMemsetAsync(workspace, 0, kErrBytes, s), "clearing the error word")) return st0;
    return build_kv2q_impl(block_idx, L, kv2q, (int*)workspace, (uint8_t*)workspace + kErrBytes, s);
}

} // extern "C"

namespace msa {

// Host checks of msa_build_kv2q_static: the same layout validation and fault hook as
// msa_build_kv2q, with a fixed scratch of scratch_bytes in place of the caller's workspace.
msa_status kv2q_static_check(const int32_t* block_idx, const msa_kv2q_layout* L, const void* kv2q,
                             size_t scratch_bytes)
{
    if (!block_idx || !L || !kv2q) return MSA_ERR_INVALID_ARG;
    if (!layout_ok(L) || !aligned(kv2q, 256) || !aligned(block_idx, 4)) return MSA_ERR_INVALID_ARG;
    if (kErrBytes + kv2q_internal_tmp(*L) > scratch_bytes) return MSA_ERR_WORKSPACE;
    if (injected("msa_build_kv2q_static")) return MSA_ERR_CUDA;
    return MSA_OK;
}

// The inversion with its error word and scan partials in `scratch` (a checked layout).
msa_status kv2q_static_run(const int32_t* block_idx, const msa_kv2q_layout* L, void* kv2q, void* scratch,
                           cudaStream_t s)
{
    if (msa_status st0 = cuda_status(cudaMemsetAsync(scratch, 0, kErrBytes, s), "clearing the error word")) return st0;
    return build_kv2q_impl(block_idx, L, kv2q, (int*)scratch, (uint8_t*)scratch + kErrBytes, s);
}

} // namespace msa

extern "C" {

// ------------------------------------------------------------------------------------ sparse prefill
static size_t partial_row_bytes(int H_q, int d_h, int k) { return (size_t)k * H_q * ((size_t)d_h * 2 + 4); }

// Attention + combine over the windows of an inversion, wins_per_pass windows per pass.
static msa_status run_passes(const uint8_t* kvb, const msa_kv2q_layout* L, int64_t N, int H_q, int H_kv, int d_h, int k,
                             const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                             int64_t wins_per_pass, int64_t rows_pass, uint16_t* o_part, float* lse_part,
                             msa_bf16* out, float* lse, void* workspace, cudaStream_t s, const int32_t* blk_tok,
                             const int32_t* row_start, const int32_t* blk_qtok = nullptr,
                             const AttnArgs* f8 = nullptr)
{
    for (int64_t w0 = 0; w0 < L->n_windows; w0 += wins_per_pass) {
        const int64_t w1 = w0 + wins_per_pass < L->n_windows ? w0 + wins_per_pass : L->n_windows;
        AttnArgs a;
        a.N = N;
        a.H_q = H_q;
        a.H_kv = H_kv;
        a.d_h = d_h;
        a.k = k;
        a.entries = (const int32_t*)(kvb + L->entries);
        a.items = (const msa_work_item*)(kvb + L->items);
        a.window_items = (const int32_t*)(kvb + L->window_items);
        a.w0 = (int)w0;
        a.w1 = (int)w1;
        a.row0 = w0 * L->window;
        a.rows_pass = rows_pass;
        a.item_counter = (int*)workspace + 4; // inside the error-word region, reset for every pass
        a.blk_tok = blk_tok;
        a.blk_qtok = blk_qtok;
        a.timeline = nullptr;
        a.timeline_tiles = 0;
        a.o_part = o_part;
        a.lse_part = lse_part;
        a.err = (int*)workspace;
        if (f8) {
            a.qs = f8->qs;
            a.ks = f8->ks;
            a.vs = f8->vs;
            a.rvs = f8->rvs;
            a.vblkmax = f8->vblkmax;
            a.sstride = f8->sstride;
            a.nb = f8->nb;
        }
        if (msa_status st1 = cuda_status(cudaMemsetAsync(a.item_counter, 0, sizeof(int), s), "clearing the work counter"))
            return st1;
        trace_begin(s);
        const cudaError_t ea = f8 ? launch_sparse_attn_fp8(a, qmap, kmap, vmap, s)
                                  : launch_sparse_attn(a, qmap, kmap, vmap, s);
        trace_end(s, MSA_KERNEL_ATTN);
        if (ea != cudaSuccess) return cuda_status(ea, "attention launch");
        CombineArgs c;
        c.row0 = a.row0;
        c.n_rows = (w1 * L->window < N ? w1 * L->window : N) - a.row0;
        c.H_q = H_q;
        c.d_h = d_h;
        c.k = k;
        c.local_of_row_div = kBk;
        c.o_part = o_part;
        c.lse_part = lse_part;
        c.nsel = nullptr;
        c.out = out;
        c.lse = lse;
        c.row_start = row_start;
        trace_begin(s);
        const cudaError_t ec = launch_combine(c, s);
        trace_end(s, MSA_KERNEL_COMBINE);
        if (ec != cudaSuccess) return cuda_status(ec, "combine launch");
    }
    return MSA_OK;
}

size_t msa_sparse_prefill_workspace_size(int64_t N, int H_q, int H_kv, int d_h, int B_k, int k,
                                         int64_t max_rows_per_pass, int internal_kv2q)
{
    msa_kv2q_layout L;
    if (msa_kv2q_layout_get(N, H_kv, B_k, k, 0, 0, &L) != MSA_OK || H_q < 1) return 0;
    int64_t rows = max_rows_per_pass <= 0 || max_rows_per_pass > N ? N : max_rows_per_pass;
    rows = (rows + L.window - 1) / L.window * L.window;
    size_t sz = kErrBytes + 512; // error word + alignment slack of the partial buffers
    if (internal_kv2q) sz += align_up(L.total_bytes, 256) + align_up(kv2q_internal_tmp(L), 256);
    sz += align_up((size_t)rows * k * H_q * d_h * 2, 256) + align_up((size_t)rows * k * H_q * 4, 256);
    return sz;
}

msa_status msa_sparse_prefill(const msa_bf16* q, const msa_bf16* kk, const msa_bf16* v, int64_t N, int H_q, int H_kv,
                              int d_h, int B_k, int k, const int32_t* block_idx, const msa_kv2q_layout* layout,
                              const void* kv2q, msa_bf16* out, float* lse, void* workspace, size_t workspace_bytes,
                              msa_stream_t stream)
{
    if (!q || !kk || !v || !block_idx || !out || !workspace || N < 1 || H_q < 1 || H_kv < 1 || d_h < 1 || k < 1)
        return MSA_ERR_INVALID_ARG;
    if ((layout == nullptr) != (kv2q == nullptr)) return MSA_ERR_INVALID_ARG;
    if (H_q % H_kv != 0) return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(kk, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(workspace, 256) ||
        (lse && !aligned(lse, 4)))
        return MSA_ERR_INVALID_ARG;
    const int G = H_q / H_kv;
    if (B_k != kBk || k > kMaxK || !(d_h == 64 || d_h == 128) || !pow2(G) || G > 128 || N > kMaxN)
        return MSA_ERR_UNSUPPORTED;
    if (layout && (!layout_ok(layout) || layout->N != N || layout->H_kv != H_kv || layout->k != k))
        return MSA_ERR_INVALID_ARG;
    if (injected("msa_sparse_prefill")) return MSA_ERR_CUDA;

    msa_kv2q_layout Lint;
    const msa_kv2q_layout* L = layout;
    uint8_t* ws = (uint8_t*)workspace;
    size_t used = kErrBytes;
    const void* kv = kv2q;
    cudaStream_t s = (cudaStream_t)stream;
    // every size check happens before anything is enqueued
    void* kvbuf = nullptr;
    void* kvtmp = nullptr;
    if (!L) {
        msa_kv2q_layout_get(N, H_kv, B_k, k, 0, 0, &Lint);
        L = &Lint;
        const size_t need = align_up(L->total_bytes, 256) + align_up(kv2q_internal_tmp(*L), 256);
        if (workspace_bytes < used + need) return MSA_ERR_WORKSPACE;
        kvbuf = ws + used;
        kvtmp = ws + used + align_up(L->total_bytes, 256);
        used += need;
        kv = kvbuf;
    }
    // rows of partials the remaining workspace holds, in whole windows
    const size_t per_row = partial_row_bytes(H_q, d_h, k);
    if (workspace_bytes <= used + 512) return MSA_ERR_WORKSPACE;
    int64_t rows_cap = (int64_t)((workspace_bytes - used - 512) / per_row);
    int64_t wins_per_pass = rows_cap / L->window;
    if (wins_per_pass < 1) return MSA_ERR_WORKSPACE;
    if (wins_per_pass > L->n_windows) wins_per_pass = L->n_windows;
    const int64_t rows_pass = wins_per_pass * L->window;
    uint16_t* o_part = (uint16_t*)(ws + used);
    float* lse_part = (float*)(ws + used + align_up((size_t)rows_pass * k * H_q * d_h * 2, 256));

    CUtensorMap qmap, kmap, vmap;
    if (!make_qmap(&qmap, q, d_h, H_q, N, G) ||
        !make_map_3d(&kmap, kk, d_h, H_kv, N, 64, 1, kBk, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_3d(&vmap, v, d_h, H_kv, N, 64, 1, kBk, CU_TENSOR_MAP_SWIZZLE_128B))
        return MSA_ERR_INVALID_ARG;

    if (msa_status st0 = cuda_status(cudaMemsetAsync(workspace, 0, kErrBytes, s), "clearing the error word")) return st0;
    if (kvbuf) {
        msa_status st = build_kv2q_impl(block_idx, L, kvbuf, (int*)workspace, kvtmp, s);
        if (st != MSA_OK) return st;
    }
    return run_passes((const uint8_t*)kv, L, N, H_q, H_kv, d_h, k, qmap, kmap, vmap, wins_per_pass, rows_pass, o_part,
                      lse_part, out, lse, workspace, s, nullptr, nullptr);
}

// ------------------------------------------------------------------------------------ FP8 main branch
msa_status msa_quantize_e4m3(const msa_bf16* x, int64_t N, int H, int d, uint8_t* codes, float* scales,
                             float* rscales, float* blkmax, msa_stream_t stream)
{
    if (!x || !codes || !scales || N < 1 || H < 1 || d < 1) return MSA_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 16) || (rscales && !aligned(rscales, 16)) ||
        (blkmax && !aligned(blkmax, 4)))
        return MSA_ERR_INVALID_ARG;
    if (!(d == 64 || d == 128) || N > kMaxN) return MSA_ERR_UNSUPPORTED;
    if (injected("msa_quantize_e4m3")) return MSA_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    QuantArgs a;
    a.x = x;
    a.N = N;
    a.nb = (int)((N + kBk - 1) / kBk);
    a.N_pad = (int64_t)a.nb * kBk;
    a.H = H;
    a.d = d;
    a.codes = codes;
    a.scales = scales;
    a.rscales = rscales;
    a.blkmax = blkmax;
    if (blkmax)
        if (msa_status st = cuda_status(cudaMemsetAsync(blkmax, 0, (size_t)H * a.nb * 4, s), "clearing blkmax"))
            return st;
    trace_begin(s);
    const cudaError_t e = launch_quantize_e4m3(a, s);
    trace_end(s, MSA_KERNEL_QUANT);
    return cuda_status(e, "quantize launch");
}

msa_status msa_sparse_prefill_fp8(const uint8_t* q8, const float* qs, const uint8_t* k8, const float* ks,
                                  const uint8_t* v8, const float* vs, const float* rvs, const float* vblkmax, int64_t N,
                                  int H_q, int H_kv, int d_h, int B_k, int k, const int32_t* block_idx,
                                  const msa_kv2q_layout* layout, const void* kv2q, msa_bf16* out, float* lse,
                                  void* workspace, size_t workspace_bytes, msa_stream_t stream)
{
    if (!q8 || !qs || !k8 || !ks || !v8 || !vs || !rvs || !vblkmax || !block_idx || !out || !workspace || N < 1 ||
        H_q < 1 || H_kv < 1 || d_h < 1 || k < 1)
        return MSA_ERR_INVALID_ARG;
    if ((layout == nullptr) != (kv2q == nullptr)) return MSA_ERR_INVALID_ARG;
    if (H_q % H_kv != 0) return MSA_ERR_INVALID_ARG;
    if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(v8, 16) || !aligned(qs, 16) || !aligned(ks, 16) ||
        !aligned(vs, 16) || !aligned(rvs, 16) || !aligned(vblkmax, 4) || !aligned(out, 16) || !aligned(workspace, 256) ||
        (lse && !aligned(lse, 4)))
        return MSA_ERR_INVALID_ARG;
    const int G = H_q / H_kv;
    if (B_k != kBk || k > kMaxK || d_h != 128 || !pow2(G) || G > 16 || N > kMaxN) return MSA_ERR_UNSUPPORTED;
    if (layout && (!layout_ok(layout) || layout->N != N || layout->H_kv != H_kv || layout->k != k))
        return MSA_ERR_INVALID_ARG;
    if (injected("msa_sparse_prefill_fp8")) return MSA_ERR_CUDA;

    msa_kv2q_layout Lint;
    const msa_kv2q_layout* L = layout;
    uint8_t* ws = (uint8_t*)workspace;
    size_t used = kErrBytes;
    const void* kv = kv2q;
    cudaStream_t s = (cudaStream_t)stream;
    void* kvbuf = nullptr;
    void* kvtmp = nullptr;
    if (!L) {
        msa_kv2q_layout_get(N, H_kv, B_k, k, 0, 0, &Lint);
        L = &Lint;
        const size_t need = align_up(L->total_bytes, 256) + align_up(kv2q_internal_tmp(*L), 256);
        if (workspace_bytes < used + need) return MSA_ERR_WORKSPACE;
        kvbuf = ws + used;
        kvtmp = ws + used + align_up(L->total_bytes, 256);
        used += need;
        kv = kvbuf;
    }
    const size_t per_row = partial_row_bytes(H_q, d_h, k);
    if (workspace_bytes <= used + 512) return MSA_ERR_WORKSPACE;
    int64_t wins_per_pass = (int64_t)((workspace_bytes - used - 512) / per_row) / L->window;
    if (wins_per_pass < 1) return MSA_ERR_WORKSPACE;
    if (wins_per_pass > L->n_windows) wins_per_pass = L->n_windows;
    const int64_t rows_pass = wins_per_pass * L->window;
    uint16_t* o_part = (uint16_t*)(ws + used);
    float* lse_part = (float*)(ws + used + align_up((size_t)rows_pass * k * H_q * d_h * 2, 256));

    CUtensorMap qmap, kmap, vmap;
    if (!make_qmap(&qmap, q8, d_h, H_q, N, G, 1) ||
        !make_map_3d(&kmap, k8, d_h, H_kv, N, 128, 1, kBk, CU_TENSOR_MAP_SWIZZLE_128B, 1) ||
        !make_map_3d(&vmap, v8, d_h, H_kv, N, 128, 1, kBk, CU_TENSOR_MAP_SWIZZLE_128B, 1))
        return MSA_ERR_INVALID_ARG;
    AttnArgs f8;
    f8.qs = qs;
    f8.ks = ks;
    f8.vs = vs;
    f8.rvs = rvs;
    f8.vblkmax = vblkmax;
    f8.nb = (int)((N + kBk - 1) / kBk);
    f8.sstride = (int64_t)f8.nb * kBk;

    if (msa_status st0 = cuda_status(cudaMemsetAsync(workspace, 0, kErrBytes, s), "clearing the error word")) return st0;
    if (kvbuf) {
        msa_status st = build_kv2q_impl(block_idx, L, kvbuf, (int*)workspace, kvtmp, s);
        if (st != MSA_OK) return st;
    }
    return run_passes((const uint8_t*)kv, L, N, H_q, H_kv, d_h, k, qmap, kmap, vmap, wins_per_pass, rows_pass, o_part,
                      lse_part, out, lse, workspace, s, nullptr, nullptr, nullptr, &f8);
}

// ------------------------------------------------------------------------------------ backward
size_t msa_sparse_backward_workspace_size(int64_t N, int H_q, int H_kv, int d_h, int B_k, int k, int d_idx,
                                          int internal_kv2q)
{
    msa_kv2q_layout L;
    if (msa_kv2q_layout_get(N, H_kv, B_k, k, 0, 0, &L) != MSA_OK || H_q < 1 || d_h < 1) return 0;
    if (d_idx != 0 && d_idx != 32 && d_idx != 64) return 0;
    size_t sz = kErrBytes; // error word and work counter
    if (internal_kv2q) sz += align_up(L.total_bytes, 256) + align_up(kv2q_internal_tmp(L), 256);
    sz += align_up((size_t)N * H_q * 4, 256);            // D = rowsum(dout * out)
    sz += align_up((size_t)N * H_q * d_h * 4, 256);      // dq accumulator
    sz += 2 * align_up((size_t)N * H_kv * d_h * 4, 256); // dk, dv accumulators
    if (d_idx) sz += align_up((size_t)N * H_kv * 4, 256) + 2 * align_up((size_t)N * H_kv * d_idx * 4, 256);
    return sz;
}

msa_status msa_sparse_backward(const msa_bf16* q, const msa_bf16* kk, const msa_bf16* v, const msa_bf16* out,
                               const float* lse, const msa_bf16* dout, int64_t N, int H_q, int H_kv, int d_h, int B_k,
                               int k, const int32_t* block_idx, const msa_kv2q_layout* layout, const void* kv2q,
                               msa_bf16* dq, msa_bf16* dk, msa_bf16* dv, const msa_bf16* q_idx, const msa_bf16* k_idx,
                               int d_idx, float kl_weight, msa_bf16* dq_idx, msa_bf16* dk_idx, float* kl,
                               void* workspace, size_t workspace_bytes, msa_stream_t stream)
{
    if (!q || !kk || !v || !out || !lse || !dout || !dq || !dk || !dv || !workspace || N < 1 || H_q < 1 || H_kv < 1 ||
        d_h < 1 || k < 1)
        return MSA_ERR_INVALID_ARG;
    if ((layout == nullptr) != (kv2q == nullptr) || (!layout && !block_idx)) return MSA_ERR_INVALID_ARG;
    if (H_q % H_kv != 0) return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(kk, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(dout, 16) ||
        !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4) || !aligned(workspace, 256))
        return MSA_ERR_INVALID_ARG;
    const int G = H_q / H_kv;
    if (B_k != kBk || k > kMaxK || !(d_h == 64 || d_h == 128) || !pow2(G) || G > 16 || N > kMaxN)
        return MSA_ERR_UNSUPPORTED;
    if (layout && (!layout_ok(layout) || layout->N != N || layout->H_kv != H_kv || layout->k != k))
        return MSA_ERR_INVALID_ARG;
    const bool with_kl = q_idx != nullptr;
    if (with_kl) {
        if (!k_idx || !dq_idx || !dk_idx || !block_idx || !aligned(q_idx, 16) || !aligned(k_idx, 16) ||
            !aligned(dq_idx, 16) || !aligned(dk_idx, 16) || (kl && !aligned(kl, 4)))
            return MSA_ERR_INVALID_ARG;
        if (d_idx != 32 && d_idx != 64) return MSA_ERR_UNSUPPORTED;
    }
    if (injected("msa_sparse_backward")) return MSA_ERR_CUDA;

    msa_kv2q_layout Lint;
    const msa_kv2q_layout* L = layout;
    uint8_t* ws = (uint8_t*)workspace;
    size_t used = kErrBytes;
    const uint8_t* kv = (const uint8_t*)kv2q;
    void* kvbuf = nullptr;
    void* kvtmp = nullptr;
    if (!L) {
        msa_kv2q_layout_get(N, H_kv, B_k, k, 0, 0, &Lint);
        L = &Lint;
        kvbuf = ws + used;
        kvtmp = ws + used + align_up(L->total_bytes, 256);
        used += align_up(L->total_bytes, 256) + align_up(kv2q_internal_tmp(*L), 256);
        kv = (const uint8_t*)kvbuf;
    }
    float* D = (float*)(ws + used);
    used += align_up((size_t)N * H_q * 4, 256);
    uint8_t* acc0 = ws + used;
    float* dq_acc = (float*)(ws + used);
    used += align_up((size_t)N * H_q * d_h * 4, 256);
    float* dk_acc = (float*)(ws + used);
    used += align_up((size_t)N * H_kv * d_h * 4, 256);
    float* dv_acc = (float*)(ws + used);
    used += align_up((size_t)N * H_kv * d_h * 4, 256);
    float *dqi_acc = nullptr, *dki_acc = nullptr, *lse_idx = nullptr;
    if (with_kl) {
        dqi_acc = (float*)(ws + used);
        used += align_up((size_t)N * H_kv * d_idx * 4, 256);
        dki_acc = (float*)(ws + used);
        used += align_up((size_t)N * H_kv * d_idx * 4, 256);
        lse_idx = (float*)(ws + used); // written before it is read: outside the cleared range
        used += align_up((size_t)N * H_kv * 4, 256);
    }
    const size_t acc_bytes = (size_t)((lse_idx ? (uint8_t*)lse_idx : ws + used) - acc0);
    if (workspace_bytes < used) return MSA_ERR_WORKSPACE;

    cudaStream_t s = (cudaStream_t)stream;
    if (msa_status st0 = cuda_status(cudaMemsetAsync(workspace, 0, kErrBytes, s), "clearing the error word")) return st0;
    if (kvbuf) {
        msa_status st = build_kv2q_impl(block_idx, L, kvbuf, (int*)workspace, kvtmp, s);
        if (st != MSA_OK) return st;
    }
    if (msa_status st1 = cuda_status(cudaMemsetAsync(acc0, 0, acc_bytes, s), "clearing the accumulators"))
        return st1;
    if (with_kl && kl)
        if (msa_status st2 = cuda_status(cudaMemsetAsync(kl, 0, (size_t)N * H_kv * 4, s), "clearing kl")) return st2;
    BwdArgs a;
    a.N = N;
    a.H_q = H_q;
    a.H_kv = H_kv;
    a.d_h = d_h;
    a.k = k;
    a.q = q;
    a.kk = kk;
    a.v = v;
    a.out = out;
    a.lse = lse;
    a.dout = dout;
    a.entries = (const int32_t*)(kv + L->entries);
    a.items = (const msa_work_item*)(kv + L->items);
    a.window_items = (const int32_t*)(kv + L->window_items);
    a.n_windows = L->n_windows;
    a.D = D;
    a.dq_acc = dq_acc;
    a.dk_acc = dk_acc;
    a.dv_acc = dv_acc;
    a.item_counter = (int*)workspace + 4; // inside the error-word region, cleared above
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.err = (int*)workspace;
    if (with_kl) {
        a.q_idx = q_idx;
        a.k_idx = k_idx;
        a.block_idx = block_idx;
        a.d_idx = d_idx;
        a.kl_weight = kl_weight;
        a.lse_idx = lse_idx;
        a.dqi_acc = dqi_acc;
        a.dki_acc = dki_acc;
        a.kl = kl;
        a.dq_idx = dq_idx;
        a.dk_idx = dk_idx;
    }
    return cuda_status(launch_backward(a, s), "backward launch");
}

// ------------------------------------------------------------------------------------ varlen prefill
} // extern "C"

namespace {

// Host-side plan of a packed batch: global block bases (key blocks of every sequence) and the index
// work items (sequence, query tile pair) in decreasing work order.
struct VarlenPlan {
    int B = 0;
    int64_t T = 0, Tk = 0, NB = 0;
    std::vector<int32_t> head; // [cu (B+1) | cu_k (B+1) | blk_base (B+1) | vitems (2 * n_vitems)]
    int n_vitems = 0;
    size_t off_cu = 0, off_cuk = 0, off_base = 0, off_items = 0, head_bytes = 0;
};

msa_status varlen_plan(const int32_t* cu, const int32_t* cu_k, int B, VarlenPlan& p)
{
    if (!cu || B < 1 || cu[0] != 0 || (cu_k && cu_k[0] != 0)) return MSA_ERR_INVALID_ARG;
    if (!cu_k) cu_k = cu;
    for (int s = 0; s < B; ++s) {
        const int32_t nq = cu[s + 1] - cu[s], nk = cu_k[s + 1] - cu_k[s];
        if (nq < 0 || nk < nq) return MSA_ERR_INVALID_ARG;       // keys cover the queries' positions
        if ((nk - nq) % kBk != 0) return MSA_ERR_UNSUPPORTED;   // cached prefix in whole blocks
    }
    p.B = B;
    p.T = cu[B];
    p.Tk = cu_k[B];
    if (p.T < 1) return MSA_ERR_INVALID_ARG;
    if (p.T > kMaxN || p.Tk > kMaxN) return MSA_ERR_UNSUPPORTED;
    std::vector<int32_t> base(B + 1, 0);
    std::vector<std::pair<int, std::pair<int, int>>> items; // (work, (s, u))
    for (int s = 0; s < B; ++s) {
        const int nq = cu[s + 1] - cu[s], nk = cu_k[s + 1] - cu_k[s];
        base[s + 1] = base[s] + (nk + kBk - 1) / kBk;
        const int t0 = (nk - nq) / kBk, n_qt = (nq + kBk - 1) / kBk;
        for (int u = 0; u < (n_qt + 1) / 2; ++u) items.push_back({t0 + 2 * u, {s, u}});
    }
    p.NB = base[B];
    std::stable_sort(items.begin(), items.end(),
                     [](const std::pair<int, std::pair<int, int>>& x, const std::pair<int, std::pair<int, int>>& y) {
                         return x.first > y.first; // most work first
                     });
    p.n_vitems = (int)items.size();
    const size_t cu_bytes = align_up((size_t)(B + 1) * 4, 16);
    p.off_cu = 0;
    p.off_cuk = cu_bytes;
    p.off_base = 2 * cu_bytes;
    p.off_items = 3 * cu_bytes;
    p.head_bytes = align_up(p.off_items + (size_t)p.n_vitems * 8, 256);
    p.head.assign(p.head_bytes / 4, 0);
    for (int s = 0; s <= B; ++s) {
        p.head[p.off_cu / 4 + s] = cu[s];
        p.head[p.off_cuk / 4 + s] = cu_k[s];
        p.head[p.off_base / 4 + s] = base[s];
    }
    for (int j = 0; j < p.n_vitems; ++j) {
        p.head[p.off_items / 4 + 2 * j] = items[j].second.first;
        p.head[p.off_items / 4 + 2 * j + 1] = items[j].second.second;
    }
    return MSA_OK;
}

// Workspace carve-up of msa_sparse_prefill_varlen; rows_pass = 0 in the plan means "size query".
struct VarlenWs {
    size_t head, row_start, row_gb0, blk_tok, blk_qtok, kv2q, kvtmp, parts, total;
    int64_t rows_pass;
    msa_kv2q_layout L;
};

msa_status varlen_ws(const VarlenPlan& p, int H_q, int H_kv, int d_h, int k, int64_t max_rows_per_pass,
                     size_t workspace_bytes, VarlenWs& w)
{
    if (msa_status st = layout_fill(p.T, H_kv, kBk, k, p.NB, 0, 0, &w.L)) return st;
    size_t off = kErrBytes;
    w.head = off;
    off += p.head_bytes;
    w.row_start = off;
    off += align_up((size_t)p.T * 4, 256);
    w.row_gb0 = off;
    off += align_up((size_t)p.T * 4, 256);
    w.blk_tok = off;
    off += align_up((size_t)p.NB * 4, 256);
    w.blk_qtok = off;
    off += align_up((size_t)p.NB * 4, 256);
    w.kv2q = off;
    off += align_up(w.L.total_bytes, 256);
    w.kvtmp = off;
    off += align_up(kv2q_internal_tmp(w.L), 256);
    w.parts = off;
    const size_t per_row = partial_row_bytes(H_q, d_h, k);
    if (workspace_bytes == 0) { // size query: room for max_rows_per_pass rows (whole windows)
        int64_t rows = max_rows_per_pass <= 0 || max_rows_per_pass > p.T ? p.T : max_rows_per_pass;
        rows = (rows + w.L.window - 1) / w.L.window * w.L.window;
        w.rows_pass = rows;
        w.total = off + 512 + align_up((size_t)rows * k * H_q * d_h * 2, 256) + align_up((size_t)rows * k * H_q * 4, 256);
        return MSA_OK;
    }
    if (workspace_bytes <= off + 512) return MSA_ERR_WORKSPACE;
    const int64_t wins = (int64_t)((workspace_bytes - off - 512) / per_row) / w.L.window;
    if (wins < 1) return MSA_ERR_WORKSPACE;
    w.rows_pass = (wins < w.L.n_windows ? wins : w.L.n_windows) * w.L.window;
    w.total = workspace_bytes;
    return MSA_OK;
}

} // namespace

extern "C" {

size_t msa_sparse_prefill_varlen_workspace_size(const int32_t* cu_seqlens, const int32_t* cu_seqlens_k, int B, int H_q,
                                                int H_kv, int d_h, int B_k, int k, int64_t max_rows_per_pass)
{
    VarlenPlan p;
    VarlenWs w;
    if (B_k != kBk || H_q < 1 || H_kv < 1 || d_h < 1 || varlen_plan(cu_seqlens, cu_seqlens_k, B, p) != MSA_OK ||
        varlen_ws(p, H_q, H_kv, d_h, k, max_rows_per_pass, 0, w) != MSA_OK)
        return 0;
    return w.total;
}

msa_status msa_sparse_prefill_varlen(const msa_bf16* q, const msa_bf16* kk, const msa_bf16* v, const msa_bf16* q_idx,
                                     const msa_bf16* k_idx, const int32_t* cu_seqlens, const int32_t* cu_seqlens_k,
                                     int B, int H_q, int H_kv,
                                     int d_h, int d_idx, int B_k, int k, int32_t* block_idx, msa_bf16* out, float* lse,
                                     void* workspace, size_t workspace_bytes, msa_stream_t stream)
{
    if (!q || !kk || !v || !q_idx || !k_idx || !block_idx || !out || !workspace || H_q < 1 || H_kv < 1 || d_h < 1 ||
        d_idx < 1 || k < 1 || H_q % H_kv != 0)
        return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(kk, 16) || !aligned(v, 16) || !aligned(q_idx, 16) || !aligned(k_idx, 16) ||
        !aligned(block_idx, 4) || !aligned(out, 16) || !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
        return MSA_ERR_INVALID_ARG;
    const int G = H_q / H_kv;
    if (B_k != kBk || k > kMaxK || !(d_h == 64 || d_h == 128) || !pow2(G) || G > 128 ||
        !(d_idx == 32 || d_idx == 64 || d_idx == 128) || H_kv > 65535)
        return MSA_ERR_UNSUPPORTED;
    VarlenPlan p;
    if (msa_status st = varlen_plan(cu_seqlens, cu_seqlens_k, B, p)) return st;
    VarlenWs w;
    if (msa_status st = varlen_ws(p, H_q, H_kv, d_h, k, 0, workspace_bytes, w)) return st;
    if (injected("msa_sparse_prefill_varlen")) return MSA_ERR_CUDA;
    const int64_t T = p.T, Tk = p.Tk;
    CUtensorMap qim, kim, qmap, kmap, vmap;
    const uint32_t box0 = d_idx < 64 ? (uint32_t)d_idx : 64u;
    const CUtensorMapSwizzle sw = d_idx == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_map_3d(&qim, q_idx, d_idx, H_kv, T, box0, 1, kBk, sw) ||
        !make_map_3d(&kim, k_idx, d_idx, H_kv, Tk, box0, 1, kBk, sw) ||
        !make_qmap(&qmap, q, d_h, H_q, T, G) ||
        !make_map_3d(&kmap, kk, d_h, H_kv, Tk, 64, 1, kBk, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_3d(&vmap, v, d_h, H_kv, Tk, 64, 1, kBk, CU_TENSOR_MAP_SWIZZLE_128B))
        return MSA_ERR_INVALID_ARG;

    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* ws = (uint8_t*)workspace;
    const int32_t* d_cu = (const int32_t*)(ws + w.head + p.off_cu);
    const int32_t* d_cuk = (const int32_t*)(ws + w.head + p.off_cuk);
    const int32_t* d_base = (const int32_t*)(ws + w.head + p.off_base);
    const int2* d_items = (const int2*)(ws + w.head + p.off_items);
    int32_t* row_start = (int32_t*)(ws + w.row_start);
    int32_t* row_gb0 = (int32_t*)(ws + w.row_gb0);
    int32_t* blk_tok = (int32_t*)(ws + w.blk_tok);
    int32_t* blk_qtok = (int32_t*)(ws + w.blk_qtok);
    if (msa_status st = cuda_status(cudaMemsetAsync(workspace, 0, kErrBytes, s), "clearing the error word")) return st;
    if (msa_status st = cuda_status(cudaMemcpyAsync(ws + w.head, p.head.data(), p.head_bytes, cudaMemcpyHostToDevice, s),
                                    "copying the batch plan"))
        return st;
    if (msa_status st = cuda_status(launch_varlen_tables(d_cu, d_cuk, d_base, B, T, (int32_t)p.NB, row_start, row_gb0,
                                                         blk_tok, blk_qtok, s),
                                    "varlen tables launch"))
        return st;
    // index branch over (sequence, tile pair) items
    IndexTopkArgs ia{q_idx, k_idx, T, H_kv, d_idx, k, block_idx, (int*)workspace};
    ia.vitems = d_items;
    ia.n_vitems = p.n_vitems;
    ia.cu = d_cu;
    ia.cu_k = d_cuk;
    trace_begin(s);
    const cudaError_t ei = launch_index_topk(ia, qim, kim, s);
    trace_end(s, MSA_KERNEL_INDEX_TOPK);
    if (ei != cudaSuccess) return cuda_status(ei, "index_topk launch");
    // inversion keyed on global blocks
    if (msa_status st = build_kv2q_impl(block_idx, &w.L, ws + w.kv2q, (int*)workspace, ws + w.kvtmp, s, row_start,
                                        row_gb0))
        return st;
    const int64_t wins_per_pass = w.rows_pass / w.L.window;
    uint16_t* o_part = (uint16_t*)(ws + w.parts);
    float* lse_part = (float*)(ws + w.parts + align_up((size_t)w.rows_pass * k * H_q * d_h * 2, 256));
    return run_passes(ws + w.kv2q, &w.L, T, H_q, H_kv, d_h, k, qmap, kmap, vmap, wins_per_pass, w.rows_pass, o_part,
                      lse_part, out, lse, workspace, s, blk_tok, row_start, blk_qtok);
}

// ------------------------------------------------------------------------------------ decode
size_t msa_sparse_decode_workspace_size(int B, int64_t L_max, int H_q, int H_kv, int d_h, int, int B_k, int k)
{
    if (B < 1 || L_max < 1 || B_k < 1 || k < 1) return 0;
    const int64_t nb_max = (L_max + B_k - 1) / B_k;
    size_t sz = kErrBytes;
    sz += align_up((size_t)B * H_kv * nb_max * 4, 256);
    sz += align_up((size_t)B * H_kv * k * 4, 256);
    sz += align_up((size_t)B * 4, 256);
    sz += align_up((size_t)B * k * H_q * d_h * 2, 256);
    sz += align_up((size_t)B * k * H_q * 4, 256);
    sz += align_up((size_t)(B + 1) * 8, 256);
    return sz;
}

msa_status msa_sparse_decode(const msa_bf16* q, const msa_bf16* q_idx, const msa_bf16* k_cache,
                             const msa_bf16* v_cache, const msa_bf16* k_idx_cache, const int32_t* lens, int B,
                             int64_t L_max, int H_q, int H_kv, int d_h, int d_idx, int B_k, int k, msa_bf16* out,
                             float* lse, int32_t* block_idx_out, void* workspace, size_t workspace_bytes,
                             msa_stream_t stream)
{
    if (!q || !q_idx || !k_cache || !v_cache || !k_idx_cache || !lens || !out || !workspace || B < 1 || L_max < 1 ||
        H_q < 1 || H_kv < 1 || d_h < 1 || d_idx < 1 || k < 1)
        return MSA_ERR_INVALID_ARG;
    if (H_q % H_kv != 0) return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(q_idx, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(k_idx_cache, 16) || !aligned(lens, 4) || !aligned(out, 16) || !aligned(workspace, 256) ||
        (lse && !aligned(lse, 4)) || (block_idx_out && !aligned(block_idx_out, 4)))
        return MSA_ERR_INVALID_ARG;
    const int G = H_q / H_kv;
    const int lanes_per_pos = H_kv * d_idx / 8;
    if (B_k != kBk || k > kMaxK || !(d_h == 64 || d_h == 128) || !pow2(G) || G > 16 ||
        !(d_idx == 32 || d_idx == 64 || d_idx == 128) || !pow2(lanes_per_pos) || lanes_per_pos > 32 ||
        L_max > kMaxN || B > 65535 || H_kv > 65535)
        return MSA_ERR_UNSUPPORTED;
    if (workspace_bytes < msa_sparse_decode_workspace_size(B, L_max, H_q, H_kv, d_h, d_idx, B_k, k))
        return MSA_ERR_WORKSPACE;
    if (injected("msa_sparse_decode")) return MSA_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* ws = (uint8_t*)workspace;
    if (msa_status st0 = cuda_status(cudaMemsetAsync(workspace, 0, kErrBytes, s), "clearing the error word")) return st0;
    const int64_t nb_max = (L_max + B_k - 1) / B_k;
    size_t off = kErrBytes;
    DecodeArgs a;
    a.q = q;
    a.q_idx = q_idx;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.k_idx_cache = k_idx_cache;
    a.lens = lens;
    a.B = B;
    a.L_max = L_max;
    a.H_q = H_q;
    a.H_kv = H_kv;
    a.d_h = d_h;
    a.d_idx = d_idx;
    a.k = k;
    a.pooled = (float*)(ws + off);
    off += align_up((size_t)B * H_kv * nb_max * 4, 256);
    a.sel = (int32_t*)(ws + off);
    off += align_up((size_t)B * H_kv * k * 4, 256);
    a.nsel = (int32_t*)(ws + off);
    off += align_up((size_t)B * 4, 256);
    a.o_part = (uint16_t*)(ws + off);
    off += align_up((size_t)B * k * H_q * d_h * 2, 256);
    a.lse_part = (float*)(ws + off);
    off += align_up((size_t)B * k * H_q * 4, 256);
    a.blk_prefix = (int64_t*)(ws + off);
    a.out = out;
    a.lse = lse;
    a.block_idx_out = block_idx_out;
    a.err = (int*)workspace;
    return cuda_status(launch_decode(a, s), "decode launch");
}

} // extern "C"
