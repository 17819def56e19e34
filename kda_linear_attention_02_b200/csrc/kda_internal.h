// kda_internal.h -- host-side launch functions shared between the libkda translation units.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kda {

// The driver's tensor-map encoder (looked up once; nullptr when the driver lacks it) (kda_chunk_bf16.cu).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Decode step (kda_decode.cu).
cudaError_t launch_decode(float* state, const void* q, const void* k, const void* v, const float* la,
                          const float* beta, void* o, int nh, int dk, int dv, bool bf16, cudaStream_t s);
// Decode step with MXFP8 q, k, v (codes + E8M0 scale arrays), bf16 o (kda_decode.cu).
cudaError_t launch_decode_mx(float* state, const void* q, const uint8_t* qs, const void* k, const uint8_t* ks,
                             const void* v, const uint8_t* vs, const float* la, const float* beta, void* o, int nh,
                             int dk, int dv, cudaStream_t s);
// Speculative decoding (kda_decode.cu): n_accept == nullptr verifies (outputs of all n_draft drafts, state
// read only); otherwise commits the first n_accept[i] drafts of every sequence into the state.
cudaError_t launch_decode_multi(float* state, const void* q, const void* k, const void* v, const float* la,
                                const float* beta, int n, int H, int n_draft, const int32_t* n_accept, void* o,
                                int dk, int dv, bool bf16, int* status, cudaStream_t s);

// Segment compose (kda_compose.cu).
cudaError_t launch_compose(const float* M, const float* Z, const int32_t* seg_cu, const float* init, int n_seqs,
                           int n_segs, int H, int dk, int dv, float* starts, float* ends, int* status,
                           cudaStream_t s);

// Optional per-kernel events of one kda_chunk_fwd call (null = not recording).
struct ChunkEvents {
    cudaEvent_t ev[4];   // before index, before prep, before state, after state
};
// Everything one chunk-path launch needs (kda_chunk_f32.cu / kda_chunk_bf16.cu).
struct ChunkArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* log_alpha;
    const float* beta;
    const void* q_scale;        // MXFP8 inputs only: E8M0 shared scales [T, H, dk / 32], [T, H, dv / 32]
    const void* k_scale;
    const void* v_scale;
    bool mx;                    // q, k, v are MXFP8 codes (bf16 path with in-kernel decode)
    const float* initial_state;
    const int32_t* cu_seqlens;
    const int32_t* cu_chunks;   // device [N+1], filled by launch_chunk_index
    int n_seqs;
    int64_t total_tokens;
    int H, dk, dv;
    int ckpt_stride;
    void* o;
    float* final_state;
    float* checkpoints;
    const int32_t* ckpt_cu;
    float* final_transition;
    float* carry;               // [N,H,dk,dv+dk] fp32 state carried between windows (or null)
    void* packets;              // window of per-(chunk, head) packets
    int2* chunk_tab;            // window of per-chunk {first token, valid tokens} (bf16 path)
    long long win_lo, win_hi;   // global chunk index window [lo, hi)
    bool multi_window;
    int* status;                // device status word
    struct ChunkEvents* events; // per-kernel timing events of this call, or null
};

// Builds cu_chunks[i] = sum_{j<i} ceil(len_j / 64) from cu_seqlens and validates the table.
cudaError_t launch_chunk_index(const int32_t* cu_seqlens, int n_seqs, int64_t total_tokens, int32_t* cu_chunks,
                               int* status, cudaStream_t s);

// fp32 path: SIMT fp32 intra-chunk prep + inter-chunk state pass.
size_t chunk_packet_bytes_f32(int dk, int dv);
cudaError_t launch_chunk_f32(const ChunkArgs& a, cudaStream_t s);

// bf16 path: tcgen05 intra-chunk prep + tcgen05 inter-chunk state pass.
size_t chunk_packet_bytes_bf16(int dk, int dv);
cudaError_t launch_chunk_bf16(const ChunkArgs& a, cudaStream_t s);

ChunkEvents* profile_slot();   // events for the current call, or null

// Diagnostics.
cudaError_t launch_selftest_wait(int limit_us, int* d_result, cudaStream_t s);
cudaError_t launch_selftest_mma_rate(int n, int k, int majors, int reps, float* cycles, int grid, int* status,
                                     cudaStream_t s);
cudaError_t launch_selftest_umma(const void* a, const void* b, float* d, int n, int flags, int* status,
                                 cudaStream_t s);

}  // namespace kda
