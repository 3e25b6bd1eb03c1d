// common.cuh -- shared definitions of the MSA CUDA library (device error word, limits, launchers).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "msa.h"

namespace msa {

// Every bounded wait gives up after this many SM clock cycles (~1 s at 2 GHz) and records
// MSA_ERR_TIMEOUT in the device error word.
constexpr long long kWaitLimit = 2000000000LL;

constexpr int kBk = 128;       // KV block size this build supports (one tensor-core tile)
constexpr int kMaxK = 16;      // largest k
constexpr int kMaxN = 1 << 21; // largest sequence length (nb <= 16384)

// Device error word: the first 16 bytes of every workspace. [0] = status code, [1] = detail.
struct ErrWord {
    int code;
    int detail;
    int pad[2];
};

__device__ __forceinline__ void report_error(int* word, int code, int detail)
{
    if (atomicCAS(word, 0, code) == 0) word[1] = detail;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline int align_up_dev(int x) { return (x + 15) & ~15; }

// Opt-in per-kernel event tracing and the launch counter (msa_trace_set / msa_launch_count).
void trace_begin(cudaStream_t s);
void trace_end(cudaStream_t s, int kernel_id);
void note_launch(int n);

// ---------------------------------------------------------------------------------------------
// launchers implemented in the .cu files
// ---------------------------------------------------------------------------------------------
struct IndexTopkArgs {
    const uint16_t* q_idx;
    const uint16_t* k_idx;
    int64_t N;
    int H_kv, d_idx, k;
    int32_t* block_idx;
    int* err;
    // packed batch of sequences (nullptr: one sequence of N rows): items are (sequence, tile pair)
    const int2* vitems = nullptr; // [n_vitems] (sequence, pair u), decreasing work first
    int n_vitems = 0;
    const int32_t* cu = nullptr;   // [B+1] first query row of each sequence
    const int32_t* cu_k = nullptr; // [B+1] first key row of each sequence (nullptr: same as cu)
};
cudaError_t launch_index_topk(const IndexTopkArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                              cudaStream_t s);

struct Kv2qArgs {
    const int32_t* block_idx;
    int64_t N;
    int H_kv, k, nb, window, chunk, n_windows;
    int32_t* offsets;
    int32_t* entries;
    msa_work_item* items;
    int32_t* window_items;
    int32_t* counts; // [H_kv][nb][n_windows]
    int32_t* bases;  // [H_kv][nb][n_windows]
    int64_t max_items;
    int32_t* scan_tmp;
    int* err;
    // packed batch (nullptr: one sequence): selections hold blocks local to the row's sequence
    const int32_t* row_start = nullptr; // [N] first row of the row's sequence
    const int32_t* row_gb0 = nullptr;   // [N] global index of the row's sequence's block 0
};
cudaError_t launch_kv2q(const Kv2qArgs& a, cudaStream_t s);
size_t kv2q_scan_tmp_bytes(int64_t n, int H_kv);
// msa_build_kv2q_static: host checks (layout, alignment, scratch size, fault hook), then the launch
// with the error word and scan partials in a fixed scratch (msa_api.cu).
msa_status kv2q_static_check(const int32_t* block_idx, const msa_kv2q_layout* L, const void* kv2q,
                             size_t scratch_bytes);
msa_status kv2q_static_run(const int32_t* block_idx, const msa_kv2q_layout* L, void* kv2q, void* scratch,
                           cudaStream_t s);

struct AttnArgs {
    int64_t N;
    int H_q, H_kv, d_h, k;
    const int32_t* entries;     // [H_kv][N*k]
    const msa_work_item* items; // work list
    const int32_t* window_items;
    int w0, w1;                 // windows of this pass
    int64_t row0;               // first row of the pass (= w0 * window)
    int64_t rows_pass;          // rows the partial buffers hold
    int* item_counter;          // work items claimed so far in this launch (zero at launch)
    const int32_t* blk_tok = nullptr;  // packed batch: first key row of each global block (nullptr: b * B_k)
    const int32_t* blk_qtok = nullptr; // packed batch: query-row coordinate of each block's first token
                                       // (differs from blk_tok when keys and queries are packed apart)
    long long* timeline;        // optional: CTA 0 records clock64 per tile event (nullptr = off)
    int timeline_tiles;         // capacity in tiles (48 event slots per tile)
    uint16_t* o_part;           // [rows][k][d_h / 16][H_q][16] bf16 (normalised partial outputs)
    float* lse_part;            // [rows][k][H_q]
    int* err;
    // FP8 main branch (the q, k, v maps then hold E4M3 codes): head-major row scales [H][sstride]
    const float* qs = nullptr;      // q scales
    const float* ks = nullptr;      // k scales
    const float* vs = nullptr;      // v scales
    const float* rvs = nullptr;     // reciprocals of the v scales
    const float* vblkmax = nullptr; // [H_kv][nb]: largest v scale of each 128-token block
    int64_t sstride = 0;            // N rounded up to whole 128-token blocks
    int nb = 0;
};

// Per-row E4M3 quantisation: x [N][H][d] bf16 -> codes [N][H][d], scales [H][N_pad] (amax / 448, 1 for
// an all-zero or padding row), rscales = 1 / scales (nullable), blkmax [H][nb] = largest scale of each
// 128-token block (nullable; zeroed by the caller).
struct QuantArgs {
    const uint16_t* x;
    int64_t N, N_pad;
    int H, d, nb;
    uint8_t* codes;
    float* scales;
    float* rscales;
    float* blkmax;
};
cudaError_t launch_quantize_e4m3(const QuantArgs& a, cudaStream_t s);
// One thread waits on a barrier phase that never completes; the wait expires after limit_cycles.
cudaError_t launch_selftest_wait(int* err, long long limit_cycles, cudaStream_t s);

cudaError_t launch_sparse_attn(const AttnArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                               const CUtensorMap& vmap, cudaStream_t s);
// The same on E4M3 codes (d_h = 128): the maps describe 8-bit tensors, a.qs .. a.vblkmax are set.
cudaError_t launch_sparse_attn_fp8(const AttnArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                                   const CUtensorMap& vmap, cudaStream_t s);

struct CombineArgs {
    int64_t row0, n_rows; // rows [row0, row0+n_rows) of the sequence
    int H_q, d_h, k;
    int64_t local_of_row_div; // B_k: n_sel(i) = min(k, i / B_k + 1)
    const uint16_t* o_part;   // [n_rows][k][H_q][d_h]
    const float* lse_part;    // [n_rows][k][H_q]
    const int32_t* nsel;      // optional per-row count of valid slots (decode), else NULL
    uint16_t* out;            // [*, H_q, d_h] rows offset by row0
    float* lse;               // nullable
    const int32_t* row_start = nullptr; // packed batch: first row of each row's sequence (local index)
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);

// Packed batch tables from cu[B+1] (query rows), cu_k[B+1] (key rows) and blk_base[B+1] (global
// block of each sequence's block 0): row_start[i], row_gb0[i] for every query row, blk_tok[gb] and
// blk_qtok[gb] for every global block.
cudaError_t launch_varlen_tables(const int32_t* cu, const int32_t* cu_k, const int32_t* blk_base, int B, int64_t T,
                                 int32_t nb_total, int32_t* row_start, int32_t* row_gb0, int32_t* blk_tok,
                                 int32_t* blk_qtok, cudaStream_t s);

struct DecodeArgs {
    const uint16_t* q;
    const uint16_t* q_idx;
    const uint16_t* k_cache;
    const uint16_t* v_cache;
    const uint16_t* k_idx_cache;
    const int32_t* lens;
    int B;
    int64_t L_max;
    int H_q, H_kv, d_h, d_idx, k;
    float* pooled;        // [B][H_kv][nb_max]
    int64_t* blk_prefix;  // [B + 1] fully visible blocks of the sequences before beta
    int32_t* sel;         // [B][H_kv][k]
    int32_t* nsel;        // [B]
    uint16_t* o_part;     // [B][k][H_q][d_h]
    float* lse_part;      // [B][k][H_q]
    uint16_t* out;
    float* lse;
    int32_t* block_idx_out;
    int* err;
};
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);

} // namespace msa
