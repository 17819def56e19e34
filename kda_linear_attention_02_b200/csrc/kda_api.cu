// kda_api.cu -- the C ABI of libkda (see include/kda.h): argument checks, workspace layout, the
// chunk-window loop and the launches.  Everything here is host logic or tiny bookkeeping kernels;
// the arithmetic of the operator lives in kda_decode.cu, kda_compose.cu, kda_chunk_f32.cu and
// kda_chunk_bf16.cu.
#include <algorithm>

#include "kda_device.cuh"
#include "kda_internal.h"

namespace kda {

__device__ int g_status = 0;
__device__ int g_selftest_result = 0;   // result slot of kda_selftest_wait_timeout

// cu_chunks[i] = sum_{j<i} ceil(len_j / 64).  Validates cu_seqlens (cu[0] = 0, non-decreasing,
// cu[N] = total_tokens); on a bad table records KDA_ERR_DEVICE_INPUT and writes an all-zero
// cu_chunks so that no chunk kernel does any work.
__global__ void __launch_bounds__(1024)
chunk_index_kernel(const int32_t* __restrict__ cu, int n, long long total, int32_t* __restrict__ cu_chunks,
                   int* status) {
    __shared__ int bad;
    __shared__ int warp_sums[32];
    __shared__ long long carry;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    if (t == 0) {
        bad = (cu[0] != 0) || (static_cast<long long>(cu[n]) != total);
        carry = 0;
    }
    __syncthreads();
    for (int i = t; i < n; i += 1024)
        if (cu[i + 1] < cu[i]) bad = 1;
    __syncthreads();
    if (bad) {
        for (int i = t; i <= n; i += 1024) cu_chunks[i] = 0;
        if (t == 0) set_status(status, KDA_ERR_DEVICE_INPUT);
        return;
    }
    if (t == 0) cu_chunks[0] = 0;
    for (int base = 0; base < n; base += 1024) {
        const int i = base + t;
        int c = 0;
        if (i < n) c = (cu[i + 1] - cu[i] + kChunk - 1) / kChunk;
        int x = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) warp_sums[w] = x;
        __syncthreads();
        if (w == 0) {
            int s = warp_sums[lane];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, s, off);
                if (lane >= off) s += y;
            }
            warp_sums[lane] = s;   // inclusive over warps
        }
        __syncthreads();
        const long long incl = carry + x + (w ? warp_sums[w - 1] : 0);
        if (i < n) cu_chunks[i + 1] = static_cast<int32_t>(incl);
        __syncthreads();
        if (t == 1023) carry = incl;
        __syncthreads();
    }
}

cudaError_t launch_chunk_index(const int32_t* cu_seqlens, int n_seqs, int64_t total_tokens, int32_t* cu_chunks,
                               int* status, cudaStream_t s) {
    chunk_index_kernel<<<1, 1024, 0, s>>>(cu_seqlens, n_seqs, total_tokens, cu_chunks, status);
    return cudaGetLastError();
}

__global__ void selftest_wait_kernel(unsigned long long limit_ns, int* result) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // nothing ever arrives on `bar`: the bounded wait must give up and report it
        const bool ok = mbar_wait(&bar, 0, nullptr, limit_ns);   // status left clear
        *result = ok ? 0 : 1;
    }
}

cudaError_t launch_selftest_wait(int limit_us, int* d_result, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(static_cast<unsigned long long>(limit_us) * 1000ull, d_result);
    return cudaGetLastError();
}

// ---- optional per-kernel timing of kda_chunk_fwd (see kda_profile_begin)
constexpr int kProfileMax = 256;
static ChunkEvents g_prof[kProfileMax];
static bool g_prof_created = false;
static thread_local int t_prof_limit = 0, t_prof_used = 0;

ChunkEvents* profile_slot() {
    if (t_prof_used >= t_prof_limit) return nullptr;
    return &g_prof[t_prof_used++];
}

}  // namespace kda

using namespace kda;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool supported(kda_dtype_t dt, int dk, int dv) {
    const bool dims = (dk == 64 || dk == 128) && (dv == 64 || dv == 128);
    if (!dims) return false;
    if (dt == KDA_F32) return true;
    if (dt == KDA_BF16 || dt == KDA_MXFP8) return dk == 128;
    return false;
}

size_t packet_bytes(kda_dtype_t dt, int dk, int dv) {
    return dt == KDA_F32 ? chunk_packet_bytes_f32(dk, dv) : chunk_packet_bytes_bf16(dk, dv);
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace layout: [cu_chunks (N+1 int32)] [carry (N*H*dk*(dv+dk) fp32, multi-window only)] [packets]
size_t index_bytes(int n_seqs) { return round256(static_cast<size_t>(n_seqs + 1) * sizeof(int32_t)); }
size_t carry_bytes(int n_seqs, int H, int dk, int dv) {
    return round256(static_cast<size_t>(n_seqs) * H * dk * (dv + dk) * sizeof(float));
}
long long chunk_upper_bound(int64_t total_tokens, int n_seqs) {
    return (total_tokens + kChunk - 1) / kChunk + n_seqs;
}

kda_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// Device address of the current device's status word.
int* status_ptr() {
    int* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_status) != cudaSuccess) return nullptr;
    return p;
}

}  // namespace

extern "C" {

const char* kda_version(void) { return "libkda 0.1 (sm_100a)"; }

const char* kda_status_string(kda_status_t st) {
    switch (st) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_ARG: return "KDA_ERR_ARG";
        case KDA_ERR_ALIGN: return "KDA_ERR_ALIGN";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
        case KDA_ERR_DEVICE_INPUT: return "KDA_ERR_DEVICE_INPUT";
    }
    return "KDA_ERR_UNKNOWN";
}

// Per window chunk: H packets and one chunk-table entry.
size_t chunk_bytes(kda_dtype_t dt, int H, int dk, int dv) {
    return static_cast<size_t>(H) * packet_bytes(dt, dk, dv) + sizeof(int2);
}

size_t kda_chunk_fwd_workspace_bytes(int64_t total_tokens, int n_seqs, int H, int dk, int dv, kda_dtype_t dt) {
    if (total_tokens < 0 || n_seqs < 0 || H <= 0 || !supported(dt, dk, dv)) return 0;
    return index_bytes(n_seqs) +
           static_cast<size_t>(chunk_upper_bound(total_tokens, n_seqs)) * chunk_bytes(dt, H, dk, dv);
}

size_t kda_chunk_fwd_min_workspace_bytes(int n_seqs, int H, int dk, int dv, kda_dtype_t dt) {
    if (n_seqs < 0 || H <= 0 || !supported(dt, dk, dv)) return 0;
    return index_bytes(n_seqs) + carry_bytes(n_seqs, H, dk, dv) + chunk_bytes(dt, H, dk, dv);
}

}  // extern "C"

namespace {

// kda_chunk_fwd and kda_chunk_fwd_mxfp8: dtype KDA_MXFP8 takes the shared-scale arrays (checked by the
// caller) and writes a bf16 o; it uses the bf16 path's packets and workspace.
kda_status_t chunk_fwd_impl(const void* q, const void* k, const void* v, const void* q_scale, const void* k_scale,
                            const void* v_scale, const float* log_alpha, const float* beta,
                            const float* initial_state, const int32_t* cu_seqlens, int n_seqs, int64_t total_tokens,
                            int H, int dk, int dv, kda_dtype_t dtype, int ckpt_stride, void* o, float* final_state,
                            float* checkpoints, const int32_t* ckpt_cu, float* final_transition, void* workspace,
                            size_t ws_bytes, kda_stream_t stream) {
    if (n_seqs < 0 || total_tokens < 0 || H <= 0 || ckpt_stride < 0) return KDA_ERR_ARG;
    if (total_tokens > 0x7fffffffLL) return KDA_ERR_ARG;   // cu_seqlens is int32
    if (!supported(dtype, dk, dv)) return KDA_ERR_UNSUPPORTED;
    if (ckpt_stride > 0 && (ckpt_stride % kChunk != 0 || !checkpoints || !ckpt_cu)) return KDA_ERR_ARG;
    if (n_seqs == 0) return KDA_OK;
    if (!cu_seqlens || !workspace) return KDA_ERR_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !o)) return KDA_ERR_ARG;
    // tiles of q, k, v, log_alpha move by TMA and states/outputs by 16-byte vectors: 16-byte alignment;
    // beta and the int32 tables are read element by element.
    const void* ptrs[] = {q, k, v, log_alpha, initial_state, o, final_state, checkpoints, final_transition};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_ALIGN;
    if ((beta && !aligned4(beta)) || !aligned4(cu_seqlens) || (ckpt_cu && !aligned4(ckpt_cu))) return KDA_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_ALIGN;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t pb = packet_bytes(dtype, dk, dv);
    const size_t ib = index_bytes(n_seqs);
    const long long ub = chunk_upper_bound(total_tokens, n_seqs);
    char* ws = static_cast<char*>(workspace);
    ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.initial_state = initial_state;
    a.q_scale = q_scale; a.k_scale = k_scale; a.v_scale = v_scale; a.mx = dtype == KDA_MXFP8;
    a.cu_seqlens = cu_seqlens; a.cu_chunks = reinterpret_cast<int32_t*>(ws); a.n_seqs = n_seqs;
    a.total_tokens = total_tokens; a.H = H; a.dk = dk; a.dv = dv; a.ckpt_stride = ckpt_stride; a.o = o;
    a.final_state = final_state; a.checkpoints = checkpoints; a.ckpt_cu = ckpt_cu;
    a.final_transition = final_transition;

    const size_t cbytes = chunk_bytes(dtype, H, dk, dv);
    long long win;   // chunks per window
    if (ws_bytes >= ib + static_cast<size_t>(ub) * cbytes) {
        win = ub > 0 ? ub : 1;
        a.carry = nullptr;
        a.packets = ws + ib;
        a.multi_window = false;
    } else {
        const size_t cb = carry_bytes(n_seqs, H, dk, dv);
        if (ws_bytes < ib + cb + cbytes) return KDA_ERR_WORKSPACE;
        win = static_cast<long long>((ws_bytes - ib - cb) / cbytes);
        a.carry = reinterpret_cast<float*>(ws + ib);
        a.packets = ws + ib + cb;
        a.multi_window = true;
    }
    // the chunk table of a window follows its packets
    a.chunk_tab = reinterpret_cast<int2*>(static_cast<char*>(a.packets) + static_cast<size_t>(win) * H * pb);
    a.status = status_ptr();
    if (!a.status) return KDA_ERR_CUDA;
    a.events = profile_slot();
    if (a.events) cudaEventRecord(a.events->ev[0], s);
    cudaError_t e = launch_chunk_index(cu_seqlens, n_seqs, total_tokens, reinterpret_cast<int32_t*>(ws), a.status, s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    long long lo = 0;
    do {
        a.win_lo = lo;
        a.win_hi = std::min(ub, lo + win);
        e = dtype == KDA_F32 ? launch_chunk_f32(a, s) : launch_chunk_bf16(a, s);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
        lo += win;
    } while (lo < ub);
    return KDA_OK;
}

}  // namespace

extern "C" {

kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v, const float* log_alpha, const float* beta,
                           const float* initial_state, const int32_t* cu_seqlens, int n_seqs, int64_t total_tokens,
                           int H, int dk, int dv, kda_dtype_t dtype, int ckpt_stride, void* o, float* final_state,
                           float* checkpoints, const int32_t* ckpt_cu, float* final_transition, void* workspace,
                           size_t ws_bytes, kda_stream_t stream) {
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_ARG;   // MXFP8 needs its scales: kda_chunk_fwd_mxfp8
    return chunk_fwd_impl(q, k, v, nullptr, nullptr, nullptr, log_alpha, beta, initial_state, cu_seqlens, n_seqs,
                          total_tokens, H, dk, dv, dtype, ckpt_stride, o, final_state, checkpoints, ckpt_cu,
                          final_transition, workspace, ws_bytes, stream);
}

kda_status_t kda_chunk_fwd_mxfp8(const uint8_t* q, const uint8_t* q_scale, const uint8_t* k, const uint8_t* k_scale,
                                 const uint8_t* v, const uint8_t* v_scale, const float* log_alpha, const float* beta,
                                 const float* initial_state, const int32_t* cu_seqlens, int n_seqs,
                                 int64_t total_tokens, int H, int dk, int dv, int ckpt_stride, void* o,
                                 float* final_state, float* checkpoints, const int32_t* ckpt_cu,
                                 float* final_transition, void* workspace, size_t ws_bytes, kda_stream_t stream) {
    if (!supported(KDA_MXFP8, dk, dv)) return KDA_ERR_UNSUPPORTED;
    if (n_seqs > 0 && total_tokens > 0) {
        if (!q_scale || !k_scale || !v_scale) return KDA_ERR_ARG;
        // one scale byte per 32 channels, read as whole rows: 4 bytes (128 channels) or 2 (64)
        if (!aligned_to(q_scale, dk / 32) || !aligned_to(k_scale, dk / 32) || !aligned_to(v_scale, dv / 32))
            return KDA_ERR_ALIGN;
    }
    return chunk_fwd_impl(q, k, v, q_scale, k_scale, v_scale, log_alpha, beta, initial_state, cu_seqlens, n_seqs,
                          total_tokens, H, dk, dv, KDA_MXFP8, ckpt_stride, o, final_state, checkpoints, ckpt_cu,
                          final_transition, workspace, ws_bytes, stream);
}

kda_status_t kda_recurrent_step(float* state, const void* q, const void* k, const void* v, const float* log_alpha,
                                const float* beta, int n, int H, int dk, int dv, kda_dtype_t dtype, void* o,
                                kda_stream_t stream) {
    if (n < 0 || H <= 0) return KDA_ERR_ARG;
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_ARG;
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_UNSUPPORTED;
    if (n == 0) return KDA_OK;
    if (!state || !q || !k || !v || !log_alpha || !beta || !o) return KDA_ERR_ARG;
    // the state moves by 16-byte vectors; the per-token inputs are read element by element
    const size_t es = dtype == KDA_BF16 ? 2 : 4;
    if (!aligned16(state) || !aligned_to(q, es) || !aligned_to(k, es) || !aligned_to(v, es) || !aligned_to(o, es) ||
        !aligned4(log_alpha) || !aligned4(beta))
        return KDA_ERR_ALIGN;
    if (static_cast<long long>(n) * H > 0x7fffffffLL) return KDA_ERR_ARG;
    return from_cuda(launch_decode(state, q, k, v, log_alpha, beta, o, n * H, dk, dv, dtype == KDA_BF16,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

kda_status_t kda_recurrent_step_mxfp8(float* state, const uint8_t* q, const uint8_t* q_scale, const uint8_t* k,
                                      const uint8_t* k_scale, const uint8_t* v, const uint8_t* v_scale,
                                      const float* log_alpha, const float* beta, int n, int H, int dk, int dv, void* o,
                                      kda_stream_t stream) {
    if (n < 0 || H <= 0) return KDA_ERR_ARG;
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_UNSUPPORTED;
    if (n == 0) return KDA_OK;
    if (!state || !q || !q_scale || !k || !k_scale || !v || !v_scale || !log_alpha || !beta || !o) return KDA_ERR_ARG;
    // the state moves by 16-byte vectors; codes and scales are read byte by byte
    if (!aligned16(state) || !aligned_to(o, 2) || !aligned4(log_alpha) || !aligned4(beta)) return KDA_ERR_ALIGN;
    if (static_cast<long long>(n) * H > 0x7fffffffLL) return KDA_ERR_ARG;
    return from_cuda(launch_decode_mx(state, q, q_scale, k, k_scale, v, v_scale, log_alpha, beta, o, n * H, dk, dv,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

// Shared argument checks of the two speculative-decoding calls.
static kda_status_t check_multi(int n, int n_draft, int H, int dk, int dv, kda_dtype_t dtype) {
    if (n < 0 || H <= 0 || n_draft <= 0) return KDA_ERR_ARG;
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_ARG;
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_UNSUPPORTED;
    if (static_cast<long long>(n) * H > 0x7fffffffLL) return KDA_ERR_ARG;
    if (static_cast<long long>(n) * n_draft * H > (1LL << 40)) return KDA_ERR_ARG;
    return KDA_OK;
}

kda_status_t kda_decode_verify(const float* state, const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta, int n, int n_draft, int H, int dk, int dv,
                               kda_dtype_t dtype, void* o, kda_stream_t stream) {
    const kda_status_t c = check_multi(n, n_draft, H, dk, dv, dtype);
    if (c != KDA_OK) return c;
    if (n == 0) return KDA_OK;
    if (!state || !q || !k || !v || !log_alpha || !beta || !o) return KDA_ERR_ARG;
    const size_t es = dtype == KDA_BF16 ? 2 : 4;
    if (!aligned16(state) || !aligned_to(q, es) || !aligned_to(k, es) || !aligned_to(v, es) || !aligned_to(o, es) ||
        !aligned4(log_alpha) || !aligned4(beta))
        return KDA_ERR_ALIGN;
    int* st = status_ptr();
    if (!st) return KDA_ERR_CUDA;
    return from_cuda(launch_decode_multi(const_cast<float*>(state), q, k, v, log_alpha, beta, n, H, n_draft, nullptr, o,
                                         dk, dv, dtype == KDA_BF16, st, reinterpret_cast<cudaStream_t>(stream)));
}

kda_status_t kda_decode_commit(float* state, const void* k, const void* v, const float* log_alpha,
                               const float* beta, const int32_t* n_accept, int n, int n_draft, int H, int dk, int dv,
                               kda_dtype_t dtype, kda_stream_t stream) {
    const kda_status_t c = check_multi(n, n_draft, H, dk, dv, dtype);
    if (c != KDA_OK) return c;
    if (n == 0) return KDA_OK;
    if (!state || !k || !v || !log_alpha || !beta || !n_accept) return KDA_ERR_ARG;
    const size_t es = dtype == KDA_BF16 ? 2 : 4;
    if (!aligned16(state) || !aligned_to(k, es) || !aligned_to(v, es) || !aligned4(log_alpha) || !aligned4(beta) ||
        !aligned4(n_accept))
        return KDA_ERR_ALIGN;
    int* st = status_ptr();
    if (!st) return KDA_ERR_CUDA;
    return from_cuda(launch_decode_multi(state, nullptr, k, v, log_alpha, beta, n, H, n_draft, n_accept, nullptr, dk,
                                         dv, dtype == KDA_BF16, st, reinterpret_cast<cudaStream_t>(stream)));
}

kda_status_t kda_segment_compose(const float* transitions, const float* zero_states, const int32_t* seg_cu,
                                 const float* init, int n_seqs, int n_segs, int H, int dk, int dv,
                                 float* start_states, float* end_states, kda_stream_t stream) {
    if (n_seqs < 0 || n_segs < 0 || H <= 0) return KDA_ERR_ARG;
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_UNSUPPORTED;
    if (n_seqs == 0) return KDA_OK;
    if (!seg_cu || (n_segs > 0 && (!transitions || !zero_states || !start_states))) return KDA_ERR_ARG;
    const void* ptrs[] = {transitions, zero_states, init, start_states, end_states};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_ALIGN;
    if (!aligned4(seg_cu)) return KDA_ERR_ALIGN;
    int* st = status_ptr();
    if (!st) return KDA_ERR_CUDA;
    return from_cuda(launch_compose(transitions, zero_states, seg_cu, init, n_seqs, n_segs, H, dk, dv, start_states,
                                    end_states, st, reinterpret_cast<cudaStream_t>(stream)));
}

kda_status_t kda_ckpt_offsets(const int32_t* host_cu_seqlens, int n, int stride, int32_t* host_ckpt_cu) {
    if (!host_cu_seqlens || !host_ckpt_cu || n < 0 || stride <= 0) return KDA_ERR_ARG;
    if (host_cu_seqlens[0] != 0) return KDA_ERR_ARG;
    int64_t acc = 0;
    host_ckpt_cu[0] = 0;
    for (int i = 0; i < n; ++i) {
        const int64_t len = static_cast<int64_t>(host_cu_seqlens[i + 1]) - host_cu_seqlens[i];
        if (len < 0) return KDA_ERR_ARG;
        acc += len / stride;
        if (acc > 0x7fffffffLL) return KDA_ERR_ARG;
        host_ckpt_cu[i + 1] = static_cast<int32_t>(acc);
    }
    return KDA_OK;
}

kda_status_t kda_get_device_status(kda_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
    int h = 0;
    if (cudaMemcpyFromSymbol(&h, g_status, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
    return static_cast<kda_status_t>(h);
}

kda_status_t kda_profile_begin(int max_calls) {
    if (max_calls < 0 || max_calls > kProfileMax) return KDA_ERR_ARG;
    if (!g_prof_created) {
        for (auto& c : g_prof)
            for (auto& ev : c.ev)
                if (cudaEventCreate(&ev) != cudaSuccess) return KDA_ERR_CUDA;
        g_prof_created = true;
    }
    t_prof_limit = max_calls;
    t_prof_used = 0;
    return KDA_OK;
}

kda_status_t kda_profile_end(float* ms_index, float* ms_prep, float* ms_state, int* n_calls) {
    if (!ms_index || !ms_prep || !ms_state || !n_calls) return KDA_ERR_ARG;
    float a = 0.f, b = 0.f, c = 0.f;
    for (int i = 0; i < t_prof_used; ++i) {
        float x = 0.f;
        if (cudaEventSynchronize(g_prof[i].ev[3]) != cudaSuccess) return KDA_ERR_CUDA;
        if (cudaEventElapsedTime(&x, g_prof[i].ev[0], g_prof[i].ev[1]) != cudaSuccess) return KDA_ERR_CUDA;
        a += x;
        if (cudaEventElapsedTime(&x, g_prof[i].ev[1], g_prof[i].ev[2]) != cudaSuccess) return KDA_ERR_CUDA;
        b += x;
        if (cudaEventElapsedTime(&x, g_prof[i].ev[2], g_prof[i].ev[3]) != cudaSuccess) return KDA_ERR_CUDA;
        c += x;
    }
    *ms_index = a; *ms_prep = b; *ms_state = c; *n_calls = t_prof_used;
    t_prof_limit = 0;
    t_prof_used = 0;
    return KDA_OK;
}

kda_status_t kda_selftest_wait_timeout(int limit_us, kda_stream_t stream) {
    if (limit_us <= 0 || limit_us > 1000000) return KDA_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int* d = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d), g_selftest_result) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaMemsetAsync(d, 0xff, sizeof(int), s) != cudaSuccess) return KDA_ERR_CUDA;
    cudaError_t e = launch_selftest_wait(limit_us, d, s);
    int h = -1;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&h, d, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    return h == 1 ? KDA_ERR_TIMEOUT : (h == 0 ? KDA_OK : KDA_ERR_CUDA);
}

kda_status_t kda_selftest_mma_rate(int n, int k, int majors, int reps, float* cycles, int grid,
                                   kda_stream_t stream) {
    if (n < 16 || n > 256 || (n % 16) != 0 || (k != 64 && k != 128) || reps <= 0 || reps > (1 << 20) || grid <= 0 ||
        !cycles)
        return KDA_ERR_ARG;
    if ((majors & ~(KDA_SELFTEST_B_MN_MAJOR | KDA_SELFTEST_A_MN_MAJOR | KDA_SELFTEST_M64)) != 0) return KDA_ERR_ARG;
    if ((majors & KDA_SELFTEST_B_MN_MAJOR) && (n % 64) != 0) return KDA_ERR_ARG;
    if (!aligned4(cycles)) return KDA_ERR_ALIGN;
    int* st = status_ptr();
    if (!st) return KDA_ERR_CUDA;
    return from_cuda(launch_selftest_mma_rate(n, k, majors, reps, cycles, grid, st,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

kda_status_t kda_selftest_umma(const void* a, const void* b, float* d, int n, int flags, kda_stream_t stream) {
    if (!a || !b || !d || n < 16 || n > 256 || (n % 16) != 0) return KDA_ERR_ARG;
    if ((flags & ~(KDA_SELFTEST_B_MN_MAJOR | KDA_SELFTEST_A_TMEM | KDA_SELFTEST_A_MN_MAJOR | KDA_SELFTEST_M64)) != 0)
        return KDA_ERR_ARG;
    if ((flags & KDA_SELFTEST_A_TMEM) && (flags & (KDA_SELFTEST_A_MN_MAJOR | KDA_SELFTEST_M64))) return KDA_ERR_ARG;
    if ((flags & KDA_SELFTEST_B_MN_MAJOR) && (n % 32) != 0) return KDA_ERR_ARG;
    if (!aligned16(a) || !aligned16(b) || !aligned16(d)) return KDA_ERR_ALIGN;
    int* st = status_ptr();
    if (!st) return KDA_ERR_CUDA;
    return from_cuda(launch_selftest_umma(a, b, d, n, flags, st, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
