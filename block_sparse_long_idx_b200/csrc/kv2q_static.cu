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

// Device address of the scratch array on the current device, looked up once per device. The
// stream must belong to that device: the address is only valid there. (In host code the array's
// name is only a host-side stand-in, not a device address.)
msa_status scratch_for_stream(cudaStream_t s, void** out)
{
    int dev = -1, sdev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return MSA_ERR_CUDA;
    }
    if (cudaStreamGetDevice(s, &sdev) != cudaSuccess) {
        cudaGetLastError();
        return MSA_ERR_INVALID_ARG;
    }
    if (sdev != dev) return MSA_ERR_INVALID_ARG; // a stream of another GPU
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
    // every host check first (nothing touches the GPU for a rejected call)
    if (msa_status st = msa::kv2q_static_check(block_idx, layout, kv2q, kStaticScratchBytes)) return st;
    cudaStream_t s = (cudaStream_t)stream;
    void* scratch = nullptr;
    if (msa_status st = scratch_for_stream(s, &scratch)) return st;
    return msa::kv2q_static_run(block_idx, layout, kv2q, scratch, s);
}
