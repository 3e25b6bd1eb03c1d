// topk.cuh -- exp-free register Top-k ("MiniMax Sparse Attention" explainer, section 05-1).
//
// Softmax preserves order, so block selection ranks the raw pooled scores directly. Each thread
// keeps the best k-1 (score, block) pairs of the blocks it has seen in a register-resident list
// sorted best-first. The list always has L = kMaxK - 1 slots; for a runtime k < kMaxK the first
// L - (k-1) slots hold sentinels (+inf, -1) that nothing can displace, so the admission test is a
// single compare against the last slot (a static register index, no local memory).
//
// Order ("a beats b"): larger score first; equal scores, lower block index first.
#pragma once
#include <cstdint>
#include <math_constants.h>

#include "common.cuh"

namespace msa {

__device__ __forceinline__ bool beats(float v1, int b1, float v2, int b2)
{
    return v1 > v2 || (v1 == v2 && b1 < b2);
}

struct TopkList {
    static constexpr int L = kMaxK - 1;
    float v[L];
    int b[L];

    // k_keep = k - 1 real slots.
    __device__ __forceinline__ void init(int k_keep)
    {
#pragma unroll
        for (int j = 0; j < L; ++j) {
            const bool sentinel = j < L - k_keep;
            v[j] = sentinel ? CUDART_INF_F : -CUDART_INF_F;
            b[j] = sentinel ? -1 : 0x7FFFFFFF;
        }
    }

    __device__ __forceinline__ bool admits(float val, int blk) const { return beats(val, blk, v[L - 1], b[L - 1]); }

    // Insert (val, blk) keeping the list sorted; the previous last entry falls off.
    __device__ __forceinline__ void insert(float val, int blk)
    {
        bool placed = false;
#pragma unroll
        for (int j = L - 1; j >= 0; --j) {
            if (!placed) {
                const bool shift = j > 0 && beats(val, blk, v[j - 1], b[j - 1]);
                if (shift) {
                    v[j] = v[j - 1];
                    b[j] = b[j - 1];
                } else {
                    v[j] = val;
                    b[j] = blk;
                    placed = true;
                }
            }
        }
    }

    __device__ __forceinline__ void offer(float val, int blk)
    {
        if (admits(val, blk)) insert(val, blk);
    }

    // offer() for a block whose index exceeds that of every listed block (a row's blocks offered in
    // ascending order): an equal score never beats a listed one, so the order test is a strict
    // greater-than, and the insertion becomes one independent select per slot (slot j takes its
    // left neighbour if val beats that, else val if val beats slot j, else keeps its entry) instead
    // of a serial shift. Sentinels (+inf) are never displaced.
    __device__ __forceinline__ void offer_ascending(float val, int blk)
    {
        if (!(val > v[L - 1])) return;
        bool c[L];
#pragma unroll
        for (int j = 0; j < L; ++j) c[j] = val > v[j];
#pragma unroll
        for (int j = L - 1; j >= 1; --j) {
            v[j] = c[j - 1] ? v[j - 1] : (c[j] ? val : v[j]);
            b[j] = c[j - 1] ? b[j - 1] : (c[j] ? blk : b[j]);
        }
        v[0] = c[0] ? val : v[0];
        b[0] = c[0] ? blk : b[0];
    }
};

// Final selection of one (row, group): the admitted blocks plus the local block, ascending,
// padded with -1, written to out[0..k).
__device__ __forceinline__ void emit_selection(const TopkList& t, int local, int k, int32_t* out)
{
    int sel[kMaxK];
#pragma unroll
    for (int j = 0; j < TopkList::L; ++j) sel[j] = (t.b[j] >= 0 && t.b[j] != 0x7FFFFFFF) ? t.b[j] : 0x7FFFFFFF;
    sel[kMaxK - 1] = local;
    // odd-even transposition sort, ascending (invalid = INT_MAX sinks to the end)
#pragma unroll
    for (int pass = 0; pass < kMaxK; ++pass) {
#pragma unroll
        for (int j = pass & 1; j + 1 < kMaxK; j += 2) {
            const int lo = min(sel[j], sel[j + 1]), hi = max(sel[j], sel[j + 1]);
            sel[j] = lo;
            sel[j + 1] = hi;
        }
    }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
        if (j < k) out[j] = sel[j] == 0x7FFFFFFF ? -1 : sel[j];
}

// Warp-shuffle merge of 32 per-lane lists into the warp's best k-1 (same order), returned in
// lane-uniform arrays best_v/best_b (entries past the found ones are (-inf, INT_MAX)).
// Each round every lane exposes its best remaining entry, a butterfly reduction finds the
// overall winner, and the owning lane pops it.
__device__ __forceinline__ void warp_merge(TopkList& t, int k_keep, float (&best_v)[kMaxK - 1],
                                           int (&best_b)[kMaxK - 1])
{
    const int lane = threadIdx.x & 31;
    int head = TopkList::L - k_keep; // first real slot of this lane's list
#pragma unroll
    for (int j = 0; j < TopkList::L; ++j) {
        best_v[j] = -CUDART_INF_F;
        best_b[j] = 0x7FFFFFFF;
    }
    for (int round = 0; round < k_keep; ++round) {
        float hv = -CUDART_INF_F;
        int hb = 0x7FFFFFFF;
#pragma unroll
        for (int j = 0; j < TopkList::L; ++j)
            if (j == head) {
                hv = t.v[j];
                hb = t.b[j];
            }
        float wv = hv;
        int wb = hb, wl = lane;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, wv, off);
            const int ob = __shfl_xor_sync(0xffffffffu, wb, off);
            const int ol = __shfl_xor_sync(0xffffffffu, wl, off);
            if (beats(ov, ob, wv, wb) || (ov == wv && ob == wb && ol < wl)) {
                wv = ov;
                wb = ob;
                wl = ol;
            }
        }
#pragma unroll
        for (int j = 0; j < TopkList::L; ++j)
            if (j == round) {
                best_v[j] = wv;
                best_b[j] = wb;
            }
        if (lane == wl) ++head;
    }
}

} // namespace msa
