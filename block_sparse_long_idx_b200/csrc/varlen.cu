// varlen.cu -- tables for a packed batch of independent sequences (cu_seqlens layout).
//
// Every sequence is its own causal problem: its rows select blocks of the sequence itself, numbered
// from 0 at the sequence's first token. Queries and keys may be packed apart (cu for the query rows,
// cu_k for the key rows): a sequence whose first len_k - len_q tokens are only in the key cache has
// its query rows at positions len_k - len_q .. len_k - 1. The kernels work on global block indices
// (sequence s's block b is global block blk_base[s] + b) and need, per query row, the query-row
// coordinate of its sequence's position 0 (row_start = cu[s] - prefix, so a row's position is
// i - row_start[i]) and the global index of its block 0, and per global block its first key row
// (blk_tok) and the query-row coordinate of its first token (blk_qtok).
#include "common.cuh"

namespace msa {

namespace {

__device__ __forceinline__ int seq_of(const int32_t* cu, int B, int64_t i) // last s with cu[s] <= i
{
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void varlen_tables_kernel(const int32_t* cu, const int32_t* cu_k, const int32_t* blk_base, int B, int64_t T,
                                     int32_t nb_total, int32_t* row_start, int32_t* row_gb0, int32_t* blk_tok,
                                     int32_t* blk_qtok)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < T; i += stride) {
        // empty sequences share their start with the next one: take the last, which owns row i
        const int s = seq_of(cu, B, i);
        const int32_t prefix = (cu_k[s + 1] - cu_k[s]) - (cu[s + 1] - cu[s]);
        row_start[i] = cu[s] - prefix;
        row_gb0[i] = blk_base[s];
    }
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < nb_total; g += stride) {
        const int s = seq_of(blk_base, B, g);
        const int32_t prefix = (cu_k[s + 1] - cu_k[s]) - (cu[s + 1] - cu[s]);
        const int32_t off = (int32_t)(g - blk_base[s]) * kBk;
        blk_tok[g] = cu_k[s] + off;
        blk_qtok[g] = cu[s] - prefix + off;
    }
}

} // namespace

cudaError_t launch_varlen_tables(const int32_t* cu, const int32_t* cu_k, const int32_t* blk_base, int B, int64_t T,
                                 int32_t nb_total, int32_t* row_start, int32_t* row_gb0, int32_t* blk_tok,
                                 int32_t* blk_qtok, cudaStream_t s)
{
    const int64_t n = T > nb_total ? T : nb_total;
    const int64_t blocks = (n + 255) / 256;
    varlen_tables_kernel<<<(int)(blocks < 4096 ? blocks : 4096), 256, 0, s>>>(cu, cu_k, blk_base, B, T, nb_total,
                                                                              row_start, row_gb0, blk_tok, blk_qtok);
    note_launch(1);
    return cudaGetLastError();
}

} // namespace msa
