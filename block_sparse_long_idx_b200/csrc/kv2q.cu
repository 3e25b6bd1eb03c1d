// kv2q.cu -- KV -> Q inversion and pre-scheduled chunking ("MiniMax Sparse Attention" explainer,
// section 05-2: each K/V block gathers the queries that selected it; hot blocks are split along the
// query dimension into chunks fanned out to different CTAs, without atomics in the attention).
//
// A stable counting sort keyed by (group r, block b), done per query window w of `window` rows:
//   1. count   : per (w, r) CTA, a shared-memory histogram of the window's selections -> counts[r][b][w]
//   2. scan    : bases[r][b][w] = exclusive prefix of counts in (r, b, w) order, relative to group r
//                (so offsets[r][b] = bases[r][b][0]); item bases = exclusive prefix of
//                ceil(counts / chunk) in (w, r, b) order
//   3. scatter : per (w, r) warp, rows in ascending order; lanes that hit the same block in one
//                step are ranked by lane (= by row) with match_any, so every list stays row-sorted
//   4. items   : (r, b, start, len) per chunk, ordered window-major; window_items[w] = first item
#include "common.cuh"

namespace msa {

namespace {

constexpr int kScanBlock = 1024; // elements per scan block (256 threads x 4)

// ------------------------------------------------------------------------------------ 1. count
__global__ void kv2q_count_kernel(Kv2qArgs a)
{
    extern __shared__ int32_t hist[];
    const int w = blockIdx.x, r = blockIdx.y;
    for (int b = threadIdx.x; b < a.nb; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const int64_t row_lo = (int64_t)w * a.window;
    const int64_t row_hi = min(a.N, row_lo + a.window);
    const int32_t* sel = a.block_idx + (int64_t)r * a.N * a.k;
    for (int64_t e = row_lo * a.k + threadIdx.x; e < row_hi * a.k; e += blockDim.x) {
        int32_t b = sel[e];
        const int64_t i = e / a.k;
        if (b < 0) continue;
        // packed batch: the selection holds a block of the row's own sequence; key on its global index
        const int64_t il = a.row_start ? i - a.row_start[i] : i;
        if (a.row_gb0) b += a.row_gb0[i];
        if (b >= a.nb || (int64_t)(b - (a.row_gb0 ? a.row_gb0[i] : 0)) * kBk > il) {
            report_error(a.err, MSA_ERR_DEVICE_CHECK, 100);
            continue;
        }
        atomicAdd(&hist[b], 1);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < a.nb; b += blockDim.x)
        a.counts[((int64_t)r * a.nb + b) * a.n_windows + w] = hist[b];
}

// ------------------------------------------------------------------------------------ 2. scans
// Generic exclusive scan of n int32 values given by a functor, in three passes.
struct CountsInRBW {
    const int32_t* counts;
    __device__ int32_t operator()(int64_t x) const { return counts[x]; }
};

struct ItemsInWRB { // value at (w, r, b) = ceil(counts[r][b][w] / chunk)
    const int32_t* counts;
    int H_kv, nb, n_windows, chunk;
    __device__ int32_t operator()(int64_t x) const
    {
        const int64_t b = x % nb, wr = x / nb;
        const int64_t r = wr % H_kv, w = wr / H_kv;
        const int32_t c = counts[(r * nb + b) * n_windows + w];
        return (c + chunk - 1) / chunk;
    }
};

__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_sums, int32_t& total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int32_t s = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        warp_sums[lane] = s; // inclusive prefix of warp sums
    }
    __syncthreads();
    total = warp_sums[(blockDim.x >> 5) - 1];
    const int32_t before = warp == 0 ? 0 : warp_sums[warp - 1];
    __syncthreads();
    return before + x - v;
}

template <class F>
__global__ void scan_partials_kernel(F f, int64_t n, int32_t* partials)
{
    __shared__ int32_t ws[32];
    const int64_t base = (int64_t)blockIdx.x * kScanBlock + threadIdx.x * 4;
    int32_t s = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        if (base + j < n) s += f(base + j);
    int32_t total;
    block_exclusive_scan(s, ws, total);
    if (threadIdx.x == 0) partials[blockIdx.x] = total;
}

__global__ void scan_partials_scan_kernel(int32_t* partials, int64_t n_blocks, int32_t* grand_total)
{
    __shared__ int32_t ws[32];
    int32_t carry = 0;
    for (int64_t c0 = 0; c0 < n_blocks; c0 += blockDim.x) {
        const int64_t i = c0 + threadIdx.x;
        const int32_t v = i < n_blocks ? partials[i] : 0;
        int32_t total;
        const int32_t ex = block_exclusive_scan(v, ws, total);
        if (i < n_blocks) partials[i] = carry + ex;
        carry += total;
    }
    if (threadIdx.x == 0 && grand_total) *grand_total = carry;
}

template <class F>
__global__ void scan_finish_kernel(F f, int64_t n, const int32_t* partials, int32_t* out)
{
    __shared__ int32_t ws[32];
    const int64_t base = (int64_t)blockIdx.x * kScanBlock + threadIdx.x * 4;
    int32_t v[4], s = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[j] = base + j < n ? f(base + j) : 0;
        s += v[j];
    }
    int32_t total;
    int32_t run = block_exclusive_scan(s, ws, total) + partials[blockIdx.x];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (base + j < n) out[base + j] = run;
        run += v[j];
    }
}

template <class F>
void exclusive_scan(F f, int64_t n, int32_t* out, int32_t* tmp, int32_t* grand_total, cudaStream_t s)
{
    const int64_t nblk = (n + kScanBlock - 1) / kScanBlock;
    scan_partials_kernel<F><<<(unsigned)nblk, 256, 0, s>>>(f, n, tmp);
    scan_partials_scan_kernel<<<1, 1024, 0, s>>>(tmp, nblk, grand_total);
    scan_finish_kernel<F><<<(unsigned)nblk, 256, 0, s>>>(f, n, tmp, out);
}

// bases (global prefix over all groups) -> group-relative bases and CSR offsets
__global__ void kv2q_group_starts_kernel(Kv2qArgs a, int32_t* group_starts)
{
    const int64_t per_group = (int64_t)a.nb * a.n_windows;
    for (int r = threadIdx.x; r < a.H_kv; r += blockDim.x) group_starts[r] = a.bases[r * per_group];
    if (threadIdx.x == 0) group_starts[a.H_kv] = group_starts[a.H_kv + 1]; // grand total was written there
}

__global__ void kv2q_relative_kernel(Kv2qArgs a, const int32_t* group_starts)
{
    const int64_t per_group = (int64_t)a.nb * a.n_windows;
    const int64_t total = per_group * a.H_kv;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < total; x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = x / per_group;
        const int32_t rel = a.bases[x] - group_starts[r];
        a.bases[x] = rel;
        const int64_t bw = x - r * per_group;
        if (bw % a.n_windows == 0) a.offsets[r * (a.nb + 1) + bw / a.n_windows] = rel;
    }
    if (blockIdx.x == 0)
        for (int r = threadIdx.x; r < a.H_kv; r += blockDim.x)
            a.offsets[(int64_t)r * (a.nb + 1) + a.nb] = group_starts[r + 1] - group_starts[r];
}

// ------------------------------------------------------------------------------------ 3. scatter
// The window's rows are split into nsub consecutive sub-ranges, one warp each. A warp first counts
// its sub-range's entries per block; the starting position of warp s in block b's list is the
// window's base for b plus the counts of warps 0 .. s-1, so the warps then scatter concurrently and
// every list stays row-sorted.
__device__ __forceinline__ int32_t scatter_block(const Kv2qArgs& a, int32_t b, int64_t i)
{
    if (b < 0) return -1;
    const int64_t il = a.row_start ? i - a.row_start[i] : i;
    const int32_t g0 = a.row_gb0 ? a.row_gb0[i] : 0;
    return (b + g0 >= a.nb || (int64_t)b * kBk > il) ? -1 : b + g0; // invalid ones: reported by the count pass
}

__global__ void kv2q_scatter_kernel(Kv2qArgs a, int nsub)
{
    extern __shared__ int32_t next_pos[]; // [nsub][nb] next write position of each warp in each block's list
    const int w = blockIdx.x, r = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t* bases = a.bases + (int64_t)r * a.nb * a.n_windows;
    const int64_t row_lo = (int64_t)w * a.window;
    const int64_t row_hi = min(a.N, row_lo + a.window);
    const int64_t sub_rows = (row_hi - row_lo + nsub - 1) / nsub;
    const int64_t my_lo = min(row_hi, row_lo + warp * sub_rows), my_hi = min(row_hi, my_lo + sub_rows);
    const int32_t* sel = a.block_idx + (int64_t)r * a.N * a.k;
    int32_t* ent = a.entries + (int64_t)r * a.N * a.k;
    const int rows_per_step = 32 / a.k;
    const unsigned lt_mask = (1u << lane) - 1u;
    const int slot = lane % a.k;
    const bool lane_used = lane < rows_per_step * a.k;
    int32_t* mine = next_pos + (int64_t)warp * a.nb;
    for (int b = threadIdx.x; b < nsub * a.nb; b += blockDim.x) next_pos[b] = 0;
    __syncthreads();
    // 1. count this warp's entries per block
    for (int64_t i0 = my_lo; i0 < my_hi; i0 += rows_per_step) {
        const int64_t i = i0 + lane / a.k;
        const int32_t b = scatter_block(a, lane_used && i < my_hi ? sel[i * a.k + slot] : -1, i);
        const unsigned peers = __match_any_sync(0xffffffffu, b);
        if (b >= 0 && (peers & lt_mask) == 0) mine[b] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // 2. starting positions: window base + counts of the earlier sub-ranges
    for (int b = threadIdx.x; b < a.nb; b += blockDim.x) {
        int32_t pos = bases[(int64_t)b * a.n_windows + w];
        for (int s2 = 0; s2 < nsub; ++s2) {
            const int32_t c = next_pos[(int64_t)s2 * a.nb + b];
            next_pos[(int64_t)s2 * a.nb + b] = pos;
            pos += c;
        }
    }
    __syncthreads();
    // 3. scatter, rows in ascending order within the sub-range
    constexpr int kAhead = 8; // selection loads in flight per lane
    for (int64_t i00 = my_lo; i00 < my_hi; i00 += (int64_t)rows_per_step * kAhead) {
        int32_t bs[kAhead];
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
            const int64_t i = i00 + (int64_t)u * rows_per_step + lane / a.k;
            bs[u] = lane_used && i < my_hi ? sel[i * a.k + slot] : -1;
        }
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
            const int64_t i = i00 + (int64_t)u * rows_per_step + lane / a.k;
            const int32_t b = scatter_block(a, bs[u], i);
            const unsigned peers = __match_any_sync(0xffffffffu, b);
            if (b >= 0) {
                const unsigned before = peers & lt_mask;
                ent[mine[b] + __popc(before)] = (int32_t)(i * a.k + slot);
                __syncwarp(peers);
                if (before == 0) mine[b] += __popc(peers);
            }
            __syncwarp();
        }
    }
}

// ------------------------------------------------------------------------------------ 4. items
__global__ void kv2q_items_kernel(Kv2qArgs a, const int32_t* item_bases, const int32_t* n_items_total)
{
    const int64_t total = (int64_t)a.n_windows * a.H_kv * a.nb;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < total; x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = x % a.nb, wr = x / a.nb;
        const int64_t r = wr % a.H_kv, w = wr / a.H_kv;
        const int64_t rbw = (r * a.nb + b) * a.n_windows + w;
        const int32_t c = a.counts[rbw];
        const int32_t base_entry = a.bases[rbw];
        int32_t it = item_bases[x];
        if (r == 0 && b == 0) a.window_items[w] = it;
        for (int32_t j = 0; j * a.chunk < c; ++j, ++it) {
            if (it >= a.max_items) {
                report_error(a.err, MSA_ERR_DEVICE_CHECK, 101);
                break;
            }
            msa_work_item item;
            item.r = (int32_t)r;
            item.b = (int32_t)b;
            item.start = base_entry + j * a.chunk;
            item.len = min(a.chunk, c - j * a.chunk);
            a.items[it] = item;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) a.window_items[a.n_windows] = *n_items_total;
}

} // namespace

size_t kv2q_scan_tmp_bytes(int64_t n, int H_kv)
{
    const int64_t nblk = (n + kScanBlock - 1) / kScanBlock;
    return align_up((align_up((size_t)nblk, 64) + (size_t)H_kv + 16) * sizeof(int32_t), 256);
}

cudaError_t launch_kv2q(const Kv2qArgs& a, cudaStream_t s)
{
    const size_t hist_bytes = (size_t)a.nb * sizeof(int32_t);
    cudaError_t e = cudaFuncSetAttribute(kv2q_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hist_bytes);
    if (e != cudaSuccess) return e;
    // scatter: up to 8 warps per (window, group), as many as their per-block positions fit in shared memory
    int nsub = (int)((200 * 1024) / hist_bytes);
    nsub = nsub < 1 ? 1 : nsub > 8 ? 8 : nsub;
    const size_t scatter_bytes = (size_t)nsub * hist_bytes;
    e = cudaFuncSetAttribute(kv2q_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scatter_bytes);
    if (e != cudaSuccess) return e;

    const int64_t n = (int64_t)a.H_kv * a.nb * a.n_windows;
    // tmp layout: [partials (nblk, padded to 64)] [group starts (H_kv + 2)] [item total]
    const int64_t nblk = (n + kScanBlock - 1) / kScanBlock;
    int32_t* partials = a.scan_tmp;
    int32_t* group_starts = a.scan_tmp + align_up((size_t)nblk, 64); // [H_kv + 2]
    int32_t* n_items_total = group_starts + a.H_kv + 4;               // [1]
    int32_t* item_bases = a.counts + n;       // second half of the counts region holds item bases

    dim3 grid_wr(a.n_windows, a.H_kv);
    kv2q_count_kernel<<<grid_wr, 256, hist_bytes, s>>>(a);
    exclusive_scan(CountsInRBW{a.counts}, n, a.bases, partials, group_starts + a.H_kv + 1, s);
    kv2q_group_starts_kernel<<<1, 256, 0, s>>>(a, group_starts);
    const int64_t nb256 = (n + 255) / 256;
    const int nsm_blocks = (int)(nb256 < 4096 ? nb256 : 4096);
    kv2q_relative_kernel<<<nsm_blocks, 256, 0, s>>>(a, group_starts);
    kv2q_scatter_kernel<<<grid_wr, 32 * nsub, scatter_bytes, s>>>(a, nsub);
    exclusive_scan(ItemsInWRB{a.counts, a.H_kv, a.nb, a.n_windows, a.chunk}, n, item_bases, partials, n_items_total,
                   s);
    kv2q_items_kernel<<<nsm_blocks, 256, 0, s>>>(a, item_bases, n_items_total);
    note_launch(11);
    return cudaGetLastError();
}

} // namespace msa
