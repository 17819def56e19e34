// kda_noalloc.cu -- kda_chunk_fwd for callers that cannot allocate device memory.
//
// Some callers of this library may not call cudaMalloc: a serving engine that hands all device
// memory to its own pool at start-up, or a host program with a fixed device-memory budget that
// forbids allocations once it is running.  Such a caller has no workspace to hand kda_chunk_fwd.
// kda_chunk_fwd_noalloc runs the same computation with its scratch (chunk index, state carried
// between chunk windows and the per-chunk packets) in one fixed array that lives in this file, so
// the call itself allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds it until
// the process exits.  Host code cannot use the array's name as a device address, so the first call
// on each device looks the address up with cudaGetSymbolAddress (with that device current) and keeps
// it; later calls reuse it.
#include <mutex>

#include "kda_device.cuh"

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(KDA_NOALLOC_SCRATCH_BYTES);
static __device__ __align__(256) unsigned char g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of this device's scratch array (looked up once per device, device current).
kda_status_t scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return KDA_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return KDA_OK;
}

}  // namespace

extern "C" kda_status_t kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* log_alpha,
                                              const float* beta, const float* initial_state,
                                              const int32_t* cu_seqlens, int n_seqs, int64_t total_tokens, int H,
                                              int dk, int dv, kda_dtype_t dtype, int ckpt_stride, void* o,
                                              float* final_state, float* checkpoints, const int32_t* ckpt_cu,
                                              float* final_transition, kda_stream_t stream) {
    // The fixed array must hold at least the chunk index, the carried states of every (sequence,
    // head) and one chunk of packets for all heads; anything larger is refused up front.
    const size_t need = kda_chunk_fwd_min_workspace_bytes(n_seqs, H, dk, dv, dtype);
    if (n_seqs > 0 && H > 0 && need == 0) return KDA_ERR_UNSUPPORTED;
    if (need > kScratchBytes) return KDA_ERR_WORKSPACE;
    void* scratch = nullptr;
    const kda_status_t st = scratch_address(&scratch);
    if (st != KDA_OK) return st;
    // Nothing in the scratch has to start at zero: every call rebuilds the chunk index and writes
    // each packet and carried state before reading it.  The chunk windows are sized to the array.
    return kda_chunk_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens, n_seqs, total_tokens, H, dk, dv,
                         dtype, ckpt_stride, o, final_state, checkpoints, ckpt_cu, final_transition, scratch,
                         kScratchBytes, stream);
}
