// kv2q_static.cu -- msa_build_kv2q_static: the KV->Q inversion with its scratch in a fixed,
// library-owned device array instead of a caller workspace, for callers that cannot allocate
// device memory themselves (see include/msa.h).
#include <mutex>

#include "common.cuh"

namespace {

// Scratch of msa_build_kv2q_static: 256-byte device error word, then the scan partials.
constexpr size_t kStaticScratchBytes = 1u << 20; // 1 MiB per GPU that loads the library
__device__ __align__(256) uint8_t g_kv2q_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.
// (In host code the array's name is only a host-side stand-in, not a device address.)
msa_status scratch_for_current_device(void** out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kv2q_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return MSA_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MSA_OK;
}

} // namespace

extern "C" msa_status msa_build_kv2q_static(const int32_t* block_idx, const msa_kv2q_layout* layout, void* kv2q,
                                            msa_stream_t stream)
{
    if (!block_idx || !layout || !kv2q) return MSA_ERR_INVALID_ARG;
    msa_kv2q_layout ref;
    if (msa_kv2q_layout_get(layout->N, layout->H_kv, layout->B_k, layout->k, layout->window, layout->chunk, &ref) !=
            MSA_OK ||
        ref.total_bytes != layout->total_bytes || ref.max_items != layout->max_items ||
        ref.entries != layout->entries || ref.items != layout->items || ref.window_items != layout->window_items ||
        ref.counts != layout->counts || ref.bases != layout->bases || ref.offsets != layout->offsets)
        return MSA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(kv2q) % 256) != 0 || (reinterpret_cast<uintptr_t>(block_idx) % 4) != 0)
        return MSA_ERR_INVALID_ARG;
    const size_t need = 256 + msa::kv2q_scan_tmp_bytes((int64_t)layout->H_kv * layout->nb * layout->n_windows,
                                                       layout->H_kv);
    if (need > kStaticScratchBytes) return MSA_ERR_WORKSPACE; // beyond the fixed 1 MiB scratch
    void* scratch = nullptr;
    if (msa_status st = scratch_for_current_device(&scratch)) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemsetAsync(scratch, 0, 256, s) != cudaSuccess) return MSA_ERR_CUDA; // error word starts at zero
    uint8_t* base = (uint8_t*)kv2q;
    msa::Kv2qArgs a;
    a.block_idx = block_idx;
    a.N = layout->N;
    a.H_kv = layout->H_kv;
    a.k = layout->k;
    a.nb = layout->nb;
    a.window = layout->window;
    a.chunk = layout->chunk;
    a.n_windows = layout->n_windows;
    a.offsets = (int32_t*)(base + layout->offsets);
    a.entries = (int32_t*)(base + layout->entries);
    a.items = (msa_work_item*)(base + layout->items);
    a.window_items = (int32_t*)(base + layout->window_items);
    a.counts = (int32_t*)(base + layout->counts);
    a.bases = (int32_t*)(base + layout->bases);
    a.max_items = layout->max_items;
    a.scan_tmp = (int32_t*)((uint8_t*)scratch + 256);
    a.err = (int*)scratch;
    return msa::launch_kv2q(a, s) == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
