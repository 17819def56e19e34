/*
 * kda.h -- C ABI of libkda: the Kimi Delta Attention (KDA) operator on one NVIDIA B200 (sm_100a).
 *
 * The operator.  KDA is Gated DeltaNet with the scalar per-head gate replaced by a per-channel gate
 * on the key dimension ("Kimi K3 구조 분석" page, key messages; llm-wiki "Kimi K3" chapter, section 1
 * "GatedDeltaNet과 KDA의 차이").  Per (sequence, head) it keeps a fixed-size state S (dk x dv) that is
 * updated once per token and read by multiplying the query into it (same chapter, section 1):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,        o_t = S_t^T q_t,
 *
 * with alpha_t = exp(max(log_alpha_t, ln 0.0067)): every step keeps at least 0.67 % of what it held
 * (orkas.ai "Kimi K3 architecture" post, section "GPU 코드 경로 하나를 없앤 하한").  There is no scale
 * on q.  A NaN log-decay is treated as the floor (fmaxf semantics).  Precondition: log_alpha <= 0 (a
 * decay in (0, 1], i.e. forgetting).  The bf16 chunk path relies on it for the in-tile bound e^80.09 of
 * the floor section; a positive log-decay is outside the contract and can give inf or NaN there with
 * no status code.
 *
 * Conventions for every entry point:
 *  - Pointers are DEVICE pointers unless the argument says "host".  The caller owns every buffer; the
 *    library never allocates device memory.  Between calls it keeps one status word per device (see
 *    kda_get_device_status) and one fixed scratch array per device that only kda_chunk_fwd_noalloc
 *    uses (KDA_NOALLOC_SCRATCH_BYTES, compiled into the library; see that entry point).
 *  - Layouts are dense row-major, token-major with heads interleaved:
 *        q, k, log_alpha: [T_tot, H, dk]     v, o: [T_tot, H, dv]     beta: [T_tot, H]
 *        states: [N, H, dk, dv] fp32 (dv contiguous)
 *    Alignment: states, checkpoints, transitions, the chunk path's q/k/v/log_alpha/o and the
 *    decode state must be 16-byte aligned (TMA tiles and 16-byte vectors); beta, the int32 tables and
 *    the decode step's per-token inputs need only their natural alignment.  The workspace must be
 *    256-byte aligned.
 *  - dtype (kda_dtype_t) is the element type of q, k, v and o (KDA_BF16, KDA_F32).  The *_mxfp8 entry
 *    points take q, k, v as MXFP8 codes with their scale arrays and write a bf16 o.  log_alpha, beta
 *    and all states are fp32 always.
 *  - Calls are asynchronous on `stream`.  Argument errors that the host can see are returned before
 *    anything is launched.  Errors that only the device can see (a bad cu_seqlens table, a bounded
 *    wait that ran out) are recorded in the per-device status word and read with
 *    kda_get_device_status; the kernels never trap.
 *  - Supported sizes: dk, dv in {64, 128} for KDA_F32; dk = 128 and dv in {64, 128} for KDA_BF16 and
 *    for kda_chunk_fwd_mxfp8; dk, dv in {64, 128} for the decode calls of every type.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* kda_stream_t;   /* same type as cudaStream_t; NULL = legacy default */

typedef enum {
    KDA_OK = 0,
    KDA_ERR_ARG = -1,          /* null pointer, bad size, non-monotone host table, ... */
    KDA_ERR_ALIGN = -2,        /* a pointer is not aligned as documented above */
    KDA_ERR_UNSUPPORTED = -3,  /* dk/dv/dtype combination not built */
    KDA_ERR_CUDA = -4,         /* a CUDA runtime call failed (launch, symbol, attribute) */
    KDA_ERR_TIMEOUT = -5,      /* device: a bounded wait inside a kernel ran out */
    KDA_ERR_WORKSPACE = -6,    /* workspace too small for even one chunk window */
    KDA_ERR_DEVICE_INPUT = -7  /* device: cu_seqlens / seg_cu / ckpt_cu inconsistent */
} kda_status_t;

/* KDA_MXFP8: MXFP8 q, k, v (kda_chunk_fwd_mxfp8 only; for the workspace queries it sizes like KDA_BF16). */
typedef enum { KDA_BF16 = 0, KDA_F32 = 1, KDA_MXFP8 = 2 } kda_dtype_t;

/* Token count of one chunk of the chunked form (fixed) and of the tiles inside it. */
#define KDA_CHUNK 64
#define KDA_TILE 16

/*
 * Workspace bytes that let kda_chunk_fwd process the whole batch in one pass.  A smaller workspace
 * (at least kda_chunk_fwd_min_workspace_bytes) makes the call process the chunks in windows, one
 * after another, carrying the state between windows; results are identical.
 */
KDA_API size_t kda_chunk_fwd_workspace_bytes(int64_t total_tokens, int n_seqs, int H, int dk, int dv,
                                     kda_dtype_t dtype);
KDA_API size_t kda_chunk_fwd_min_workspace_bytes(int n_seqs, int H, int dk, int dv, kda_dtype_t dtype);

/*
 * Chunked (prefill) form over a packed batch of N sequences.
 *
 * The sequences are packed along the token axis; cu_seqlens (device, int32 [N+1], cu[0] = 0,
 * non-decreasing, cu[N] = total_tokens) gives their offsets.  Each sequence is cut into chunks of
 * KDA_CHUNK tokens; inside a chunk the cumulative log-decay is anchored at 16-token tile boundaries
 * so that the inverse decay inside a tile stays below e^80.09 and the diagonal tiles use the same
 * dense bf16 tensor-core product as all other tiles (orkas.ai post, decay-floor section).  The
 * intra-chunk system (I + strict_tril(beta K Gamma K^T))^-1 is solved by blocked forward
 * substitution over 16x16 tiles, and the state is carried across chunks in fp32.
 *
 *   initial_state   [N,H,dk,dv] fp32, or NULL for zero.
 *   o               [T_tot,H,dv] of `dtype` (written for every token).
 *   final_state     [N,H,dk,dv] fp32, or NULL.
 *   ckpt_stride     0 = no checkpoints, else a positive multiple of KDA_CHUNK (512 for the prefix
 *                   cache of the orkas.ai post's serving section: hashes every 512 tokens, sparse
 *                   state checkpoints at hash ends).  Checkpoint j (1-based) of sequence i is the state
 *                   after j*ckpt_stride tokens, stored at checkpoints[ckpt_cu[i] + j - 1]
 *                   ([*,H,dk,dv] fp32); ckpt_cu is the device copy of the table that
 *                   kda_ckpt_offsets fills.  When the stride divides len_i the last checkpoint equals
 *                   final_state.
 *   final_transition [N,H,dk,dk] fp32 or NULL: prod_t (I - beta_t k_t k_t^T) Diag(alpha_t) over the
 *                   sequence (the "cumulative transition" of the sequence-split paragraph of the
 *                   orkas.ai serving section; input of kda_segment_compose).
 *   workspace       device scratch of ws_bytes (see above), 256-byte aligned; contents on entry are
 *                   ignored.
 * Resuming from a checkpoint: run the suffix [b, len) with initial_state = the checkpoint at b; when b
 * is a multiple of KDA_CHUNK the chunk grid coincides with that of the unsplit run.
 */
KDA_API kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v,
                           const float* log_alpha, const float* beta,
                           const float* initial_state,
                           const int32_t* cu_seqlens, int n_seqs, int64_t total_tokens,
                           int H, int dk, int dv, kda_dtype_t dtype,
                           int ckpt_stride,
                           void* o, float* final_state,
                           float* checkpoints, const int32_t* ckpt_cu,
                           float* final_transition,
                           void* workspace, size_t ws_bytes, kda_stream_t stream);

/*
 * kda_chunk_fwd with MXFP8 q, k and v.  The til.kil9.dev "Kimi K3 기술 보고서" post (deployment
 * paragraph) says the model was trained quantisation-aware with MXFP8 activations, so the projections
 * that feed KDA may arrive in that form.  The format is that of the OCP Microscaling Formats (MX) v1.0
 * specification: each (token, head) row of q, k or v is cut into blocks of 32 consecutive channels; a
 * block holds 32 FP8 E4M3 codes and one E8M0 shared scale X = 2^(e - 127), and element i is X * E4M3(i).
 *
 *   q, k        [T_tot,H,dk] uint8 E4M3 codes, 16-byte aligned      q_scale, k_scale  [T_tot,H,dk/32] uint8
 *   v           [T_tot,H,dv] uint8 E4M3 codes, 16-byte aligned      v_scale           [T_tot,H,dv/32] uint8
 *   the scale arrays are aligned to dk/32 (q_scale, k_scale) and dv/32 (v_scale) bytes.
 *   o           [T_tot,H,dv] bf16.
 * Everything else (log_alpha, beta, states, checkpoints, transition, workspace, window processing, errors)
 * is as for kda_chunk_fwd with dtype KDA_BF16, and so are the supported sizes (dk = 128, dv in {64, 128}).
 * The codes are decoded in the kernel that reads them; the values are exact (E4M3 has 4 significant bits)
 * as long as X * E4M3 stays inside the fp32 range, so the results equal kda_chunk_fwd's on the decoded
 * values given as bf16.  NaN inputs are outside the contract: a NaN code (E4M3 S.1111.111) or a NaN
 * scale (0xFF) gives NaN results.
 */
KDA_API kda_status_t kda_chunk_fwd_mxfp8(const uint8_t* q, const uint8_t* q_scale,
                           const uint8_t* k, const uint8_t* k_scale,
                           const uint8_t* v, const uint8_t* v_scale,
                           const float* log_alpha, const float* beta,
                           const float* initial_state,
                           const int32_t* cu_seqlens, int n_seqs, int64_t total_tokens,
                           int H, int dk, int dv, int ckpt_stride,
                           void* o, float* final_state,
                           float* checkpoints, const int32_t* ckpt_cu,
                           float* final_transition,
                           void* workspace, size_t ws_bytes, kda_stream_t stream);

/*
 * kda_chunk_fwd without a workspace argument, for callers that may not allocate device memory (a
 * serving engine that gives all device memory to its own pool at start-up, or a program with a
 * fixed device-memory budget that forbids allocations while running).  The pages have no
 * counterpart to this entry point; it is library plumbing.
 *
 * Arguments, layouts and results are those of kda_chunk_fwd.  The scratch is one array of
 * KDA_NOALLOC_SCRATCH_BYTES (64 MiB) compiled into the library: every GPU that loads the library
 * holds it until the process exits.  The chunks are processed in windows sized to that array.
 * A batch whose minimum scratch (kda_chunk_fwd_min_workspace_bytes: chunk index, the carried state
 * of every (sequence, head), one chunk of packets) exceeds it is refused with KDA_ERR_WORKSPACE;
 * at dk = dv = 128 and H = 32 that allows up to 493 (sequence, head) pairs, e.g. 15 sequences of 32 heads.
 * The first call on each device looks the array's device address up (with that device current)
 * and keeps it; make that first call before any stream capture.  All calls share the one array and
 * it keeps the last call's contents (nothing in it needs to start at zero): calls that may overlap
 * on the GPU -- on different streams, or from different host threads -- race and must not be issued.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (64u << 20)
KDA_API kda_status_t kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                   const float* log_alpha, const float* beta,
                                   const float* initial_state,
                                   const int32_t* cu_seqlens, int n_seqs, int64_t total_tokens,
                                   int H, int dk, int dv, kda_dtype_t dtype,
                                   int ckpt_stride,
                                   void* o, float* final_state,
                                   float* checkpoints, const int32_t* ckpt_cu,
                                   float* final_transition, kda_stream_t stream);

/*
 * One recurrent (decode) step for n sequences x H heads, state updated in place: the fixed-size
 * state of the llm-wiki chapter's section 1 (O(1) memory per token).  state [n,H,dk,dv] fp32;
 * q, k [n,H,dk], v [n,H,dv] of `dtype`; log_alpha [n,H,dk] fp32; beta [n,H] fp32; o [n,H,dv] of
 * `dtype`.  Memory-bound: each call reads and writes the whole state once.
 */
KDA_API kda_status_t kda_recurrent_step(float* state, const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta,
                                int n, int H, int dk, int dv, kda_dtype_t dtype,
                                void* o, kda_stream_t stream);

/*
 * kda_recurrent_step with MXFP8 q, k and v (the format of kda_chunk_fwd_mxfp8: E4M3 codes, one E8M0 scale
 * per 32 consecutive channels of a (sequence, head) row).  q, k: [n,H,dk] uint8 codes with q_scale,
 * k_scale [n,H,dk/32]; v: [n,H,dv] codes with v_scale [n,H,dv/32]; o: [n,H,dv] bf16; everything else and
 * the supported sizes as kda_recurrent_step.  The codes are decoded exactly, so the results equal
 * kda_recurrent_step's with the decoded values given as bf16.
 */
KDA_API kda_status_t kda_recurrent_step_mxfp8(float* state, const uint8_t* q, const uint8_t* q_scale,
                           const uint8_t* k, const uint8_t* k_scale, const uint8_t* v,
                           const uint8_t* v_scale, const float* log_alpha, const float* beta,
                           int n, int H, int dk, int dv, void* o, kda_stream_t stream);

/*
 * Speculative decoding (orkas.ai "Kimi K3 architecture" post, section "비용은 서빙 스택에서
 * 돌아옵니다", speculative-decoding item).  The recurrent state is updated in place, so a rejected
 * draft token cannot be rolled back.  Instead the caller keeps the drafts' projected inputs, which
 * are far smaller than the state, and the state is rebuilt on chip from them.  Two calls:
 *
 *   kda_decode_verify  outputs of all n_draft draft tokens of every sequence, each o_d = S_d^T q_d
 *                      with S_d the state after drafts 1..d applied to `state`; `state` is read once
 *                      and never written (the recurrence of kda_recurrent_step, token after token);
 *   kda_decode_commit  the state after the first n_accept[i] drafts of sequence i, written in place
 *                      (one read and one write of the state; none at all when n_accept[i] = 0).
 *
 * Layouts: the drafts of sequence i are rows i*n_draft + d (d = 0..n_draft-1) of token-major arrays:
 *   q, k [n*n_draft, H, dk] and v [n*n_draft, H, dv] of `dtype`; log_alpha [n*n_draft, H, dk] fp32;
 *   beta [n*n_draft, H] fp32; o [n*n_draft, H, dv] of `dtype`;
 *   state [n, H, dk, dv] fp32 (16-byte aligned); n_accept: device int32 [n], each in 0..n_draft.
 * Supported: dk, dv in {64, 128}; n_draft >= 1.  Host-detectable errors return before any launch.
 * q, k, v and log_alpha need element alignment only; when all four start on 16-byte boundaries the
 * first four drafts' inputs are copied into the kernel's shared memory ahead of the state (faster).
 * A sequence whose n_accept is out of range keeps its state unchanged and sets the status word to
 * KDA_ERR_DEVICE_INPUT (read it with kda_get_device_status); the other sequences are committed.
 * Applying commit with n_accept[i] = a gives, bit for bit, the state of a consecutive
 * kda_recurrent_step calls on the same inputs, and verify gives their outputs.
 */
KDA_API kda_status_t kda_decode_verify(const float* state, const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta,
                               int n, int n_draft, int H, int dk, int dv, kda_dtype_t dtype,
                               void* o, kda_stream_t stream);
KDA_API kda_status_t kda_decode_commit(float* state, const void* k, const void* v,
                               const float* log_alpha, const float* beta, const int32_t* n_accept,
                               int n, int n_draft, int H, int dk, int dv, kda_dtype_t dtype,
                               kda_stream_t stream);

/*
 * Segment composition (orkas.ai serving section, sequence split): each segment s of a sequence is
 * summarised by its cumulative transition M_s [dk,dk] and its zero-start final state Z_s [dk,dv]
 * (both from kda_chunk_fwd run on the segment from a zero state with final_transition set).  An
 * exclusive prefix scan X_0 = init, X_{s+1} = M_s X_s + Z_s recovers every segment's start state.
 *   transitions  [S,H,dk,dk] fp32;  zero_states [S,H,dk,dv] fp32  (S = total segments)
 *   seg_cu       device int32 [n_seqs+1]: segments of sequence i are seg_cu[i] .. seg_cu[i+1]-1
 *   init         [n_seqs,H,dk,dv] fp32 or NULL (zero)
 *   start_states [S,H,dk,dv] fp32 (X_s of each segment);  end_states [n_seqs,H,dk,dv] or NULL.
 */
KDA_API kda_status_t kda_segment_compose(const float* transitions, const float* zero_states,
                                 const int32_t* seg_cu, const float* init,
                                 int n_seqs, int n_segs, int H, int dk, int dv,
                                 float* start_states, float* end_states, kda_stream_t stream);

/*
 * Prefix reuse bookkeeping (orkas.ai "Kimi K3 architecture" post, section "비용은 서빙 스택에서
 * 돌아옵니다", prefix-reuse item).  Half of the cache is per-token pages (full-attention layers) and half
 * one fixed-size recurrent state per request (KDA layers); a cached prefix is usable only where both
 * can be restored at the same boundary.  The granularities are decoupled: a hash every 512 tokens,
 * allocation in units of 1024-6144 tokens, and recurrent-state checkpoints kept sparsely at some hash
 * ends.  These host-only calls keep that directory; the checkpoint states themselves live in a device
 * pool [n_slots, H, dk, dv] fp32 owned by the caller, filled from kda_chunk_fwd's checkpoints and
 * passed back to it as initial_state when a request resumes.
 *
 * kda_prefix_block_hashes: chained 64-bit FNV-1a hashes of the full 512-token blocks of a token
 *   sequence: hash[i] = FNV-1a over the 8 little-endian bytes of hash[i-1] (seed for i = 0) followed
 *   by the 4 little-endian bytes of each token of block i, so hash[i] identifies tokens
 *   [0, 512 (i+1)).  tokens: host int32 [n_tokens]; hashes: host uint64 [n_tokens / 512].  Returns
 *   the number of full blocks (the partial tail block is not hashed), or -1 on a bad argument.
 *
 * kda_prefix_cache_create: a directory of at most max_blocks block hashes and n_slots checkpoint
 *   slots; checkpoints are planned every unit_blocks blocks (2..12: 1024-6144 tokens) and at the last
 *   full block of a request.  Least-recently-used entries are evicted (a block entry takes its slot
 *   with it; a slot can also be taken from an older entry that keeps its hash).  Every call takes one
 *   lock, so several host threads may share a directory.
 *
 * A slot is in one of three states: free, PENDING (handed out by kda_prefix_cache_insert, its state
 *   not yet copied) or COMMITTED (kda_prefix_cache_commit was called after the copy).  Independently a
 *   slot is PINNED while a lookup that named it has not been released.  Lookups only return committed
 *   slots; eviction and slot reuse only touch committed, unpinned slots.  So a resume point is never a
 *   slot whose copy may still be in flight, and a slot never changes under a request that resumes from
 *   it.  The copies themselves are asynchronous GPU work: commit a slot once the copy is ordered before
 *   every later reader (e.g. after synchronising its stream, or when all work runs on one stream), and
 *   release a pin once the kernel that read the slot is done with it (same rule).
 *
 * kda_prefix_cache_lookup: matched_blocks = the length of the request's leading run of cached
 *   hashes; resume_blocks = the deepest block end <= matched_blocks whose state is committed (0 if
 *   none) and resume_slot its slot (-1 if none).  The request restarts at token 512 * resume_blocks
 *   with the slot's state.  Touches the matched entries and pins resume_slot (if any) until
 *   kda_prefix_cache_release.
 *
 * kda_prefix_cache_plan: the block ends e (resume_blocks < e <= n_blocks, ascending) after which a
 *   request should store its state: multiples of unit_blocks, and n_blocks itself.  Writes at most
 *   max_out of them and returns how many there are (-1 on a bad argument).
 *
 * kda_prefix_cache_insert: records the request's n_blocks hashes and, for each planned end ends[i],
 *   writes out_slots[i]: a slot (>= 0, now PENDING) into which the caller copies the state after
 *   512 * ends[i] tokens and then commits; KDA_PREFIX_STORED if that block end already has a
 *   checkpoint slot (nothing to copy); KDA_PREFIX_NO_SLOT if every slot is busy or was used by this
 *   request.  A new slot is a free one, else one taken from the least recently used committed,
 *   unpinned checkpoint outside this request.
 *
 * kda_prefix_cache_commit: marks the given slots (out_slots of an insert; negative entries are
 *   skipped) as holding their states.  kda_prefix_cache_abort gives pending slots back instead (their
 *   copies will not happen; committed slots in the list are left alone).  kda_prefix_cache_release
 *   ends one pin of a slot returned by a lookup (a negative slot is accepted and ignored).
 */
#define KDA_PREFIX_BLOCK 512
#define KDA_PREFIX_NO_SLOT (-1)
#define KDA_PREFIX_STORED (-2)
typedef struct kda_prefix_cache kda_prefix_cache;
KDA_API int64_t kda_prefix_block_hashes(const int32_t* tokens, int64_t n_tokens, uint64_t seed, uint64_t* hashes);
KDA_API kda_status_t kda_prefix_cache_create(int64_t max_blocks, int n_slots, int unit_blocks,
                                     kda_prefix_cache** out);
KDA_API void kda_prefix_cache_destroy(kda_prefix_cache* cache);
KDA_API kda_status_t kda_prefix_cache_lookup(kda_prefix_cache* cache, const uint64_t* hashes, int64_t n_blocks,
                                     int64_t* matched_blocks, int64_t* resume_blocks, int32_t* resume_slot);
KDA_API int64_t kda_prefix_cache_plan(const kda_prefix_cache* cache, int64_t n_blocks, int64_t resume_blocks,
                              int64_t* out_ends, int64_t max_out);
KDA_API kda_status_t kda_prefix_cache_insert(kda_prefix_cache* cache, const uint64_t* hashes, int64_t n_blocks,
                                     const int64_t* ends, int64_t n_ends, int32_t* out_slots);
KDA_API kda_status_t kda_prefix_cache_commit(kda_prefix_cache* cache, const int32_t* slots, int64_t n);
KDA_API kda_status_t kda_prefix_cache_abort(kda_prefix_cache* cache, const int32_t* slots, int64_t n);
KDA_API kda_status_t kda_prefix_cache_release(kda_prefix_cache* cache, int32_t slot);
KDA_API kda_status_t kda_prefix_cache_stats(const kda_prefix_cache* cache, int64_t* n_blocks_cached,
                                    int32_t* n_slots_used);

/*
 * Host-only, pure: checkpoint offsets for kda_chunk_fwd's sparse state checkpoints (orkas.ai "Kimi K3
 * architecture" post, section "비용은 서빙 스택에서 돌아옵니다", prefix-reuse item: states are kept
 * only at some 512-token hash ends, so each sequence stores floor(len / stride) of them and the
 * sequences' checkpoints are packed one after another).  host_ckpt_cu[0] = 0 and
 * host_ckpt_cu[i+1] = host_ckpt_cu[i] + floor(len_i / stride) with len_i from host_cu_seqlens
 * (host int32 [n+1]).  Returns KDA_ERR_ARG on a bad stride or a decreasing table.
 */
KDA_API kda_status_t kda_ckpt_offsets(const int32_t* host_cu_seqlens, int n, int stride,
                              int32_t* host_ckpt_cu);

/* Synchronises `stream`, returns the current device's status word (KDA_OK if no kernel recorded an
 * error) and clears it. */
KDA_API kda_status_t kda_get_device_status(kda_stream_t stream);

/* Human-readable name of a status code (static string). */
KDA_API const char* kda_status_string(kda_status_t status);

/* Version string of the library build. */
KDA_API const char* kda_version(void);

/*
 * Per-kernel timing of kda_chunk_fwd (measurement plumbing, no KDA arithmetic).  After
 * kda_profile_begin(max_calls), the next max_calls calls of kda_chunk_fwd on this thread record CUDA
 * events on their stream around each of their kernels (chunk index, intra-chunk prep, inter-chunk
 * state).  kda_profile_end synchronises those events, writes the summed milliseconds of each kernel
 * over the recorded calls and the number of recorded calls, and stops recording.  The events are
 * created once per process (no device memory is allocated).
 */
KDA_API kda_status_t kda_profile_begin(int max_calls);
KDA_API kda_status_t kda_profile_end(float* ms_index, float* ms_prep, float* ms_state, int* n_calls);

/*
 * Diagnostics (no KDA arithmetic).
 *  kda_selftest_wait_timeout: launches one tiny kernel that waits on an mbarrier nothing will
 *  complete, with a wait limit of limit_us microseconds; returns KDA_ERR_TIMEOUT when the bounded
 *  wait ran out as designed (and leaves the status word clear).  Shows on a live GPU that the
 *  kernels' waits end without a fault.
 *  kda_selftest_umma: one 128 x n x 64 bf16 tcgen05 product D = A B^T through the same shared-memory
 *  descriptors, TMEM allocation and load path the chunk kernels use. a [128,64], b [n,64] bf16
 *  row-major (device), d [128,n] fp32 (device); n in {16, 32, ..., 256}.  flags: KDA_SELFTEST_B_MN_MAJOR
 *  stages B MN-major in 64-column blocks instead of K-major (then n must be a multiple of 32; a last
 *  32-column part fills half a block, as the state pass's 32-column slices do); KDA_SELFTEST_A_TMEM reads A
 *  from tensor memory (row m in lane m, two bf16 per 32-bit column), the operand form the segment
 *  compose uses, instead of shared memory; KDA_SELFTEST_A_MN_MAJOR stages A in shared memory MN-major
 *  (two 64-row blocks); KDA_SELFTEST_M64 issues the product with M = 64 (rows 0..63 of A), and d then
 *  receives all 128 TMEM lanes of the accumulator as the hardware placed them.  A_TMEM together with
 *  A_MN_MAJOR or M64, or any other flag bit: KDA_ERR_ARG.
 */
#define KDA_SELFTEST_B_MN_MAJOR 1
#define KDA_SELFTEST_A_TMEM 2
#define KDA_SELFTEST_A_MN_MAJOR 4
#define KDA_SELFTEST_M64 8
/*
 *  kda_selftest_mma_rate: the tensor-core rate of one product shape as the chunk kernels issue it:
 *  128 x n x k bf16 (k in {64, 128}, n in {16, ..., 256}), fp32 accumulator in TMEM.  majors:
 *  KDA_SELFTEST_B_MN_MAJOR stages B MN-major (then n a multiple of 64), KDA_SELFTEST_A_MN_MAJOR stages
 *  A MN-major; both K-major when 0; KDA_SELFTEST_M64 times M = 64 instead of 128; any other bit:
 *  KDA_ERR_ARG.  `grid` CTAs (one per SM when grid <= the SM count),
 *  each with one issuing thread, time `reps` products back to back and then `reps` products each
 *  waited for before the next, with the SM clock.  cycles (device, [grid][2] fp32) receives the SM
 *  cycles per product in the two modes (-1 if a bounded wait ran out).  FLOP per cycle per SM of a
 *  mode is 2 * 128 * n * k / cycles.
 */
KDA_API kda_status_t kda_selftest_mma_rate(int n, int k, int majors, int reps, float* cycles, int grid,
                                           kda_stream_t stream);
KDA_API kda_status_t kda_selftest_wait_timeout(int limit_us, kda_stream_t stream);
KDA_API kda_status_t kda_selftest_umma(const void* a, const void* b, float* d, int n, int flags,
                                       kda_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* KDA_H_ */
