// backward.cuh -- launchers of the main-branch backward (gradients in q, k, v with the selected
// sets held fixed).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "msa.h"

namespace msa {

struct BwdArgs {
    int64_t N;
    int H_q, H_kv, d_h, k;
    const uint16_t* q;    // [N, H_q, d_h] bf16
    const uint16_t* kk;   // [N, H_kv, d_h] bf16
    const uint16_t* v;    // [N, H_kv, d_h] bf16
    const uint16_t* out;  // [N, H_q, d_h] bf16, the forward's output
    const float* lse;     // [N, H_q], the forward's log-sum-exp (units of the scaled logits)
    const uint16_t* dout; // [N, H_q, d_h] bf16, upstream gradient
    const int32_t* entries;     // kv2q entries [H_kv][N*k] (i*k + slot)
    const msa_work_item* items; // kv2q work list
    const int32_t* window_items;
    int n_windows;
    float* D;      // [N, H_q] workspace: dout . out
    float* dq_acc; // [N, H_q, d_h] fp32 accumulators (zeroed before the launch)
    float* dk_acc; // [N, H_kv, d_h]
    float* dv_acc; // [N, H_kv, d_h]
    int* item_counter; // work items claimed so far (zero at launch)
    uint16_t* dq;  // [N, H_q, d_h] bf16 results
    uint16_t* dk;  // [N, H_kv, d_h]
    uint16_t* dv;  // [N, H_kv, d_h]
    int* err;
    // index-branch KL alignment, fused into the same pass (q_idx == nullptr: skipped)
    const uint16_t* q_idx = nullptr;     // [N, H_kv, d_idx] bf16
    const uint16_t* k_idx = nullptr;     // [N, H_kv, d_idx] bf16
    const int32_t* block_idx = nullptr;  // [H_kv, N, k] selections
    int d_idx = 0;                       // 32 or 64
    float kl_weight = 1.f;               // gradients of kl_weight * sum of KL(i, r)
    float* lse_idx = nullptr;            // [N, H_kv] workspace: log-sum-exp of the index scores over T
    float* dqi_acc = nullptr;            // [N, H_kv, d_idx] fp32 accumulators (zeroed before the launch)
    float* dki_acc = nullptr;
    float* kl = nullptr;                 // [N, H_kv] KL(i, r) (zeroed before the launch), or nullptr
    uint16_t* dq_idx = nullptr;          // [N, H_kv, d_idx] bf16 results
    uint16_t* dk_idx = nullptr;
};

// D = rowsum(dout * out) (and, with the KL part, the index log-sum-exp over each row's token set);
// the KV-outer gradient kernel; the fp32 -> bf16 conversion of the gradients. The accumulators
// (and kl) must be zero before the first.
cudaError_t launch_backward(const BwdArgs& a, cudaStream_t s);

} // namespace msa
