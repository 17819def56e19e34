// kda_decode.cu -- recurrent KDA steps (decode): one step in place, and the two halves of speculative
// decoding (verify drafts without touching the state; commit the accepted prefix).
//
// The fixed-size state of the llm-wiki "Kimi K3" chapter (section 1: S updated per token, the query
// multiplied into S, O(1) memory) with the per-channel decay of section "GatedDeltaNet과 KDA의 차이"
// and the 0.67 % retention floor of the orkas.ai "Kimi K3 architecture" post (decay-floor section):
//
//   a = exp(max(log_alpha, ln 0.0067));  p = (Diag(a) S)^T k;  u = beta (v - p);
//   S <- Diag(a) S + k u^T;              o = S^T q = (Diag(a) S)^T q + u (k . q)
//
// HBM-bound (about 1.75 flop/byte): a kernel streams each (sequence, head) state once in with 128-bit
// loads, keeps it in registers across the column reductions and rank-1 updates of every token it
// applies, and (when the state changes) streams it once out.
//
// Speculative decoding (orkas.ai post, section "비용은 서빙 스택에서 돌아옵니다", speculative-decoding
// item): the state is updated in place, so a rejected draft cannot be undone; the projected inputs of
// the drafts, far smaller than the state, are kept instead and the state is rebuilt on chip.
//   verify: outputs of all n_draft drafts from the committed state, which is read and never written;
//   commit: the state after the first n_accept[i] drafts of sequence i, written once (nothing moves
//           when n_accept[i] = 0).
#include "kda_device.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

// NT threads over a DK x DV state block: thread t holds float4 column group t % CG of the RPT
// consecutive rows (t / CG) RPT .. (t / CG) RPT + RPT - 1, so the per-row weights of a token come
// as 16-byte shared loads.  The column sums run over the same row groups in the same order whenever RG
// (and so RPT) is the same, so a 128-thread CTA over 64 columns reduces exactly like a 256-thread CTA
// over 128 columns.
template <int DK, int DV, int NT>
struct DecodeTiling {
    static constexpr int CG = DV / 4;     // float4 column groups
    static constexpr int RG = NT / CG;    // row groups
    static constexpr int RPT = DK / RG;   // state rows per thread
    static_assert(RG * CG == NT && RPT * RG == DK && DV <= NT, "tiling");
};

// Per-token staging, double-buffered by token parity so that token t + 1 can be staged while slower
// threads still read token t's values.
template <int DK, int DV, int NT>
struct DecodeSmem {
    float a[2][DK], k[2][DK], q[2][DK], ak[2][DK], aq[2][DK], v[2][DV], u[2][DV], beta[2];
    float4 red[2][DecodeTiling<DK, DV, NT>::RG][DecodeTiling<DK, DV, NT>::CG];
    float kq;
};

// One token's inputs as this thread loads them (element t of each vector; DK, DV <= NT).
struct TokenIn {
    float la, k, q, v, beta;
};

// Element i of a token vector: of type T, or (MX) an MXFP8 code with the scale of its 32-element block
// (E4M3 codes, E8M0 scales: OCP Microscaling Formats v1.0), decoded exactly.
template <typename T, bool MX>
__device__ __forceinline__ float in_value(const void* __restrict__ p, const uint8_t* __restrict__ scale, int i) {
    if constexpr (MX) return mx8_value(static_cast<const uint8_t*>(p)[i], scale[i >> 5]);
    else return to_f32(static_cast<const T*>(p)[i]);
}
// p advanced by n elements (bytes for MX codes)
template <typename T, bool MX>
__device__ __forceinline__ const void* in_at(const void* p, size_t n) {
    return static_cast<const char*>(p) + n * (MX ? 1 : sizeof(T));
}

template <typename T, int DK, int DV, bool OUT, bool MX = false>
__device__ __forceinline__ void load_token(TokenIn& x, const void* __restrict__ q, const void* __restrict__ k,
                                           const void* __restrict__ v, const float* __restrict__ la,
                                           const float* __restrict__ beta, const uint8_t* __restrict__ qs = nullptr,
                                           const uint8_t* __restrict__ ks = nullptr,
                                           const uint8_t* __restrict__ vs = nullptr) {
    const int t = threadIdx.x;
    if (t < DK) {
        x.la = la[t];
        x.k = in_value<T, MX>(k, ks, t);
        if (OUT) x.q = in_value<T, MX>(q, qs, t);
    }
    if (t < DV) x.v = in_value<T, MX>(v, vs, t);
    if (t == 0) x.beta = *beta;
}

template <int DK, int DV, int NT, bool OUT>
__device__ __forceinline__ void stage_token(DecodeSmem<DK, DV, NT>& sh, int par, const TokenIn& x) {
    const int t = threadIdx.x;
    if (t < DK) {
        const float a = __expf(floor_log_decay(x.la));
        sh.a[par][t] = a;
        sh.k[par][t] = x.k;
        sh.ak[par][t] = a * x.k;   // the row weights of the two column sums, formed once per row
        if (OUT) {
            sh.q[par][t] = x.q;
            sh.aq[par][t] = a * x.q;
        }
    }
    if (t < DV) sh.v[par][t] = x.v;
    if (t == 0) sh.beta[par] = x.beta;
}

// One token applied to the register-held state s (thread t holds rows rg + r RG, columns 4 cg ..),
// its inputs staged in sh[par] and made visible by a barrier.  OUT: also o = S_t^T q for this token.
// update = false skips the rank-1 update (the output needs only the column sums and u).
template <typename T, int DK, int DV, int NT, bool OUT>
__device__ __forceinline__ void token_step(float4 (&s)[DecodeTiling<DK, DV, NT>::RPT], DecodeSmem<DK, DV, NT>& sh,
                                           int par, T* __restrict__ o, bool update = true) {
    using DT = DecodeTiling<DK, DV, NT>;
    constexpr int CG = DT::CG, RG = DT::RG, RPT = DT::RPT;
    const int t = threadIdx.x, cg = t % CG, rg = t / CG;
    // column sums against alpha k and alpha q, two lanes per packed fp32 FMA
    float2 pk01 = make_float2(0.f, 0.f), pk23 = pk01, pq01 = pk01, pq23 = pk01;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg * RPT + r;
        const float ak = sh.ak[par][i];
        pk01 = __ffma2_rn(make_float2(ak, ak), make_float2(s[r].x, s[r].y), pk01);
        pk23 = __ffma2_rn(make_float2(ak, ak), make_float2(s[r].z, s[r].w), pk23);
        if (OUT) {
            const float aq = sh.aq[par][i];
            pq01 = __ffma2_rn(make_float2(aq, aq), make_float2(s[r].x, s[r].y), pq01);
            pq23 = __ffma2_rn(make_float2(aq, aq), make_float2(s[r].z, s[r].w), pq23);
        }
    }
    const float4 pk = make_float4(pk01.x, pk01.y, pk23.x, pk23.y);
    const float4 pq = make_float4(pq01.x, pq01.y, pq23.x, pq23.y);
    sh.red[0][rg][cg] = pk;
    if (OUT) {
        sh.red[1][rg][cg] = pq;
        if (t < 32) {
            float kq = 0.f;
            for (int i = t; i < DK; i += 32) kq = fmaf(sh.k[par][i], sh.q[par][i], kq);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
            if (t == 0) sh.kq = kq;
        }
    }
    __syncthreads();

    if (t < DV) {
        const int j = t;
        const float* red0 = reinterpret_cast<const float*>(sh.red[0]);
        float p = 0.f;
#pragma unroll
        for (int g = 0; g < RG; ++g) p += red0[g * DV + j];
        const float u = sh.beta[par] * (sh.v[par][j] - p);
        sh.u[par][j] = u;
        if (OUT) {
            const float* red1 = reinterpret_cast<const float*>(sh.red[1]);
            float pqj = 0.f;
#pragma unroll
            for (int g = 0; g < RG; ++g) pqj += red1[g * DV + j];
            o[j] = from_f32<T>(fmaf(u, sh.kq, pqj));
        }
    }
    __syncthreads();
    if (!update) return;

    const float4 u4 = reinterpret_cast<const float4*>(sh.u[par])[cg];
    const float2 u01 = make_float2(u4.x, u4.y), u23 = make_float2(u4.z, u4.w);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg * RPT + r;
        const float a = sh.a[par][i], kk = sh.k[par][i];
        const float2 a2 = make_float2(a, a), k2 = make_float2(kk, kk);
        const float2 s01 = __ffma2_rn(a2, make_float2(s[r].x, s[r].y), __fmul2_rn(k2, u01));
        const float2 s23 = __ffma2_rn(a2, make_float2(s[r].z, s[r].w), __fmul2_rn(k2, u23));
        s[r] = make_float4(s01.x, s01.y, s23.x, s23.y);
    }
}

// k . q of one token from its staged k and q (thread t < 32 sums elements t, t + 32, .. with fmaf, then
// a butterfly over the warp), as token_step forms it; lane 0's value is the one used.
template <int DK>
__device__ __forceinline__ float token_kq(const float* __restrict__ kk, const float* __restrict__ qq, int lane) {
    float kq = 0.f;
    for (int i = lane; i < DK; i += 32) kq = fmaf(kk[i], qq[i], kq);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    return kq;
}

// token_step for the speculative kernels: the same arithmetic in the same order, arranged for a chain of
// drafts.  k . q comes ready in *kq (formed ahead, for a preloaded draft) unless kq_here, when warp 0
// forms it as token_step does; with OUT the output's column sums run on threads DV .. 2 DV - 1 beside u's on threads
// 0 .. DV - 1, and those threads form o = u (k . q) + (Diag(a) S)^T q after the second barrier.
template <typename T, int DK, int DV, int NT, bool OUT>
__device__ __forceinline__ void draft_step(float4 (&s)[DecodeTiling<DK, DV, NT>::RPT], DecodeSmem<DK, DV, NT>& sh,
                                           int par, float* kq, bool kq_here, T* __restrict__ o, bool update) {
    using DT = DecodeTiling<DK, DV, NT>;
    constexpr int CG = DT::CG, RG = DT::RG, RPT = DT::RPT;
    static_assert(!OUT || NT >= 2 * DV, "threads for both reductions");
    const int t = threadIdx.x, cg = t % CG, rg = t / CG;
    float2 pk01 = make_float2(0.f, 0.f), pk23 = pk01, pq01 = pk01, pq23 = pk01;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg * RPT + r;
        const float ak = sh.ak[par][i];
        pk01 = __ffma2_rn(make_float2(ak, ak), make_float2(s[r].x, s[r].y), pk01);
        pk23 = __ffma2_rn(make_float2(ak, ak), make_float2(s[r].z, s[r].w), pk23);
        if (OUT) {
            const float aq = sh.aq[par][i];
            pq01 = __ffma2_rn(make_float2(aq, aq), make_float2(s[r].x, s[r].y), pq01);
            pq23 = __ffma2_rn(make_float2(aq, aq), make_float2(s[r].z, s[r].w), pq23);
        }
    }
    sh.red[0][rg][cg] = make_float4(pk01.x, pk01.y, pk23.x, pk23.y);
    if (OUT) {
        sh.red[1][rg][cg] = make_float4(pq01.x, pq01.y, pq23.x, pq23.y);
        if (kq_here && t < 32) {
            const float v = token_kq<DK>(sh.k[par], sh.q[par], t);
            if (t == 0) *kq = v;
        }
    }
    __syncthreads();

    float pqj = 0.f;
    if (t < DV) {
        const float* red0 = reinterpret_cast<const float*>(sh.red[0]);
        float p = 0.f;
#pragma unroll
        for (int g = 0; g < RG; ++g) p += red0[g * DV + t];
        sh.u[par][t] = sh.beta[par] * (sh.v[par][t] - p);
    } else if (OUT && t < 2 * DV) {
        const float* red1 = reinterpret_cast<const float*>(sh.red[1]);
#pragma unroll
        for (int g = 0; g < RG; ++g) pqj += red1[g * DV + t - DV];
    }
    __syncthreads();
    if (OUT && t >= DV && t < 2 * DV) o[t - DV] = from_f32<T>(fmaf(sh.u[par][t - DV], *kq, pqj));
    if (!update) return;

    const float4 u4 = reinterpret_cast<const float4*>(sh.u[par])[cg];
    const float2 u01 = make_float2(u4.x, u4.y), u23 = make_float2(u4.z, u4.w);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg * RPT + r;
        const float a = sh.a[par][i], kk = sh.k[par][i];
        const float2 a2 = make_float2(a, a), k2 = make_float2(kk, kk);
        const float2 s01 = __ffma2_rn(a2, make_float2(s[r].x, s[r].y), __fmul2_rn(k2, u01));
        const float2 s23 = __ffma2_rn(a2, make_float2(s[r].z, s[r].w), __fmul2_rn(k2, u23));
        s[r] = make_float4(s01.x, s01.y, s23.x, s23.y);
    }
}

// MX: q, k, v are MXFP8 codes with their scale arrays (q_scale, k_scale [n, H, dk / 32], v_scale
// [n, H, dv / 32]) and T is the type of o (bf16).
template <typename T, int DK, int DV, bool MX>
__global__ void __launch_bounds__(256, 2)
decode_step_kernel(float* __restrict__ state, const void* __restrict__ q, const void* __restrict__ k,
                   const void* __restrict__ v, const uint8_t* __restrict__ q_scale,
                   const uint8_t* __restrict__ k_scale, const uint8_t* __restrict__ v_scale,
                   const float* __restrict__ log_alpha, const float* __restrict__ beta, T* __restrict__ o) {
    using DT = DecodeTiling<DK, DV, 256>;
    __shared__ DecodeSmem<DK, DV, 256> sh;
    grid_dependency_wait();   // the state (and inputs) come from earlier launches
    const int head = blockIdx.x;   // sequence * H + h
    const int t = threadIdx.x, cg = t % DT::CG, rg = t / DT::CG;
    float4* S = reinterpret_cast<float4*>(state + static_cast<size_t>(head) * DK * DV);
    float4 s[DT::RPT];
    const size_t hk = static_cast<size_t>(head) * DK, hv = static_cast<size_t>(head) * DV;
    TokenIn x;
    if constexpr (MX) {
        // the token's bytes are loaded first, ahead of the 64 KiB state stream in the load queue, and
        // decoded once the state loads have been issued
        const uint8_t* qc = static_cast<const uint8_t*>(q) + hk;
        const uint8_t* kc = static_cast<const uint8_t*>(k) + hk;
        const uint8_t* vc = static_cast<const uint8_t*>(v) + hv;
        uint32_t rq = 0, rk = 0, rqs = 0, rks = 0, rv = 0, rvs = 0;
        if (t < DK) {
            x.la = log_alpha[hk + t];
            rk = kc[t];
            rks = k_scale[hk / 32 + (t >> 5)];
            rq = qc[t];
            rqs = q_scale[hk / 32 + (t >> 5)];
        }
        if (t < DV) {
            rv = vc[t];
            rvs = v_scale[hv / 32 + (t >> 5)];
        }
        if (t == 0) x.beta = beta[head];
        asm volatile("" ::: "memory");
#pragma unroll
        for (int r = 0; r < DT::RPT; ++r) s[r] = __ldcs(S + (rg * DT::RPT + r) * DT::CG + cg);
        if (t < DK) {
            x.k = mx8_value(rk, rks);
            x.q = mx8_value(rq, rqs);
        }
        if (t < DV) x.v = mx8_value(rv, rvs);
    } else {
#pragma unroll
        for (int r = 0; r < DT::RPT; ++r) s[r] = __ldcs(S + (rg * DT::RPT + r) * DT::CG + cg);
        load_token<T, DK, DV, true>(x, in_at<T, false>(q, hk), in_at<T, false>(k, hk), in_at<T, false>(v, hv),
                                    log_alpha + hk, beta + head);
    }
    stage_token<DK, DV, 256, true>(sh, 0, x);
    __syncthreads();
    token_step<T, DK, DV, 256, true>(s, sh, 0, o + hv);
#pragma unroll
    for (int r = 0; r < DT::RPT; ++r) __stcs(S + (rg * DT::RPT + r) * DT::CG + cg, s[r]);
}

// Draft inputs are token-major per sequence: token (i, d) of sequence i at row i * n_draft + d of
// [n * n_draft, H, .] arrays.  VERIFY: all n_draft tokens, outputs written, state read only.
// Otherwise (commit): the first n_accept[i] tokens, state written back; no outputs.
// Columns of the state are independent in every step (p, u and o are per column; k . q is recomputed),
// so a CTA takes one 64-column slice (blockIdx.y) with 256 * 64 / DV threads: the row groups, and so the
// reduction order, are those of decode_step_kernel, and the results equal consecutive single steps bit
// for bit.  At DV = 128 the smaller CTAs (128 threads) keep more state loads in flight per SM while
// others apply their tokens.
constexpr int kSpecSlice = 64;
template <int DV>
__host__ __device__ constexpr int spec_threads() { return 256 * kSpecSlice / DV; }
template <typename T, int DK, int DV, bool VERIFY>
__global__ void __launch_bounds__(spec_threads<DV>(), 1024 / spec_threads<DV>() / 2)
decode_multi_kernel(float* __restrict__ state, const T* __restrict__ q, const T* __restrict__ k,
                    const T* __restrict__ v, const float* __restrict__ log_alpha, const float* __restrict__ beta,
                    int H, int n_draft, const int32_t* __restrict__ n_accept, T* __restrict__ o, bool pre16,
                    int* status) {
    constexpr int DVS = kSpecSlice;
    static_assert(DV % DVS == 0, "slice");
    constexpr int NT = spec_threads<DV>();
    using DT = DecodeTiling<DK, DVS, NT>;
    static_assert(DT::RG == DecodeTiling<DK, DV, 256>::RG, "same row groups as the single step");
    __shared__ DecodeSmem<DK, DVS, NT> sh;
    grid_dependency_wait();   // the state, counts and drafts come from earlier launches
    const int head = blockIdx.x;   // sequence * H + h
    const int seq = head / H, h = head % H, j0 = blockIdx.y * DVS;
    const int t = threadIdx.x, cg = t % DT::CG, rg = t / DT::CG;
    int steps = n_draft;
    if (!VERIFY) {
        steps = n_accept[seq];
        if (steps < 0 || steps > n_draft) {   // the state of this sequence is left as it was
            if (t == 0 && h == 0 && blockIdx.y == 0) set_status(status, KDA_ERR_DEVICE_INPUT);
            return;
        }
        if (steps == 0) return;
    }
    auto row_of = [&](int d) { return (static_cast<size_t>(seq) * n_draft + d) * H + h; };
    // The inputs of the first kPre drafts go to shared memory by 16-byte asynchronous copies, issued ahead
    // of the state stream, so that no draft waits for a global load; later drafts (n_draft > kPre) are
    // loaded into registers while the one before is applied.
    constexpr int kPre = 4;
    __shared__ __align__(16) float pre_la[kPre][DK];
    __shared__ __align__(16) T pre_k[kPre][DK];
    __shared__ __align__(16) T pre_q[kPre][DK];
    __shared__ __align__(16) T pre_v[kPre][DVS];
    const int npre = !pre16 ? 0 : (steps < kPre ? steps : kPre);   // pre16: q, k, v, log_alpha 16-byte aligned
    {
        constexpr int CLA = DK * 4 / 16, CK = DK * static_cast<int>(sizeof(T)) / 16,
                      CV = DVS * static_cast<int>(sizeof(T)) / 16;
        constexpr int CPD = CLA + CK * (VERIFY ? 2 : 1) + CV;   // 16-byte chunks per draft
        for (int e = t; e < npre * CPD; e += NT) {
            const int d = e / CPD;
            int c = e % CPD;
            const size_t row = row_of(d);
            if (c < CLA) {
                cp_async16(&pre_la[d][4 * c], log_alpha + row * DK + 4 * c);
            } else if ((c -= CLA) < CK) {
                cp_async16(&pre_k[d][c * 16 / sizeof(T)], k + row * DK + c * 16 / sizeof(T));
            } else if ((c -= CK) < CV) {
                cp_async16(&pre_v[d][c * 16 / sizeof(T)], v + row * DV + j0 + c * 16 / sizeof(T));
            } else {
                c -= CV;
                cp_async16(&pre_q[d][c * 16 / sizeof(T)], q + row * DK + c * 16 / sizeof(T));
            }
        }
    }
    float beta_pre = 0.f;   // thread d < npre: beta of draft d
    if (t < npre) beta_pre = beta[row_of(t)];
    asm volatile("" ::: "memory");
    // state rows are DV wide; this CTA's float4 column groups start at j0
    float4* S = reinterpret_cast<float4*>(state + static_cast<size_t>(head) * DK * DV + j0);
    float4 s[DT::RPT];
#pragma unroll
    for (int r = 0; r < DT::RPT; ++r) s[r] = __ldcs(S + (rg * DT::RPT + r) * (DV / 4) + cg);
    cp_async_wait_all();
    __shared__ float pre_beta[kPre];
    if (t < npre) pre_beta[t] = beta_pre;
    __syncthreads();
    TokenIn x;
    auto load = [&](TokenIn& x, int d) {
        if (d < npre) {   // this thread's elements of a preloaded draft
            if (t < DK) {
                x.la = pre_la[d][t];
                x.k = to_f32(pre_k[d][t]);
                if (VERIFY) x.q = to_f32(pre_q[d][t]);
            }
            if (t < DVS) x.v = to_f32(pre_v[d][t]);
            if (t == 0) x.beta = pre_beta[d];
        } else {
            const size_t row = row_of(d);
            load_token<T, DK, DVS, VERIFY>(x, VERIFY ? q + row * DK : nullptr, k + row * DK, v + row * DV + j0,
                                           log_alpha + row * DK, beta + row);
        }
    };
    // k . q of preloaded draft d, formed once by warp d (the other drafts' in their own step); read after
    // the barriers ahead of each draft's output
    __shared__ float pre_kq[kPre];
    static_assert(NT / 32 >= kPre, "a warp per preloaded draft");
    if (VERIFY && (t >> 5) < npre) {
        const int d = t >> 5, lane = t & 31;
        float kf[DK / 32], qf[DK / 32];
#pragma unroll
        for (int m = 0; m < DK / 32; ++m) {
            kf[m] = to_f32(pre_k[d][lane + 32 * m]);
            qf[m] = to_f32(pre_q[d][lane + 32 * m]);
        }
        float kq = 0.f;
#pragma unroll
        for (int m = 0; m < DK / 32; ++m) kq = fmaf(kf[m], qf[m], kq);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (lane == 0) pre_kq[d] = kq;
    }
    load(x, 0);
    stage_token<DK, DVS, NT, VERIFY>(sh, 0, x);
    for (int d = 0; d < steps; ++d) {
        const int par = d & 1;
        if (d + 1 < steps) load(x, d + 1);
        __syncthreads();   // token d staged (and every reader of the other half is past token d - 1)
        // verify discards the state: the last draft needs its output only
        draft_step<T, DK, DVS, NT, VERIFY>(s, sh, par, d < npre ? &pre_kq[d] : &sh.kq, d >= npre,
                                           VERIFY ? o + row_of(d) * DV + j0 : nullptr, !VERIFY || d + 1 < steps);
        if (d + 1 < steps) stage_token<DK, DVS, NT, VERIFY>(sh, par ^ 1, x);
    }
    if (!VERIFY) {
#pragma unroll
        for (int r = 0; r < DT::RPT; ++r) __stcs(S + (rg * DT::RPT + r) * (DV / 4) + cg, s[r]);
    }
}

// Consecutive decode launches are chained (programmatic stream serialization): the next kernel's
// blocks may be scheduled while the previous one drains and wait (grid_dependency_wait) before any
// memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <typename T, int DK, int DV, bool MX = false>
cudaError_t launch_decode_t(float* state, const void* q, const void* k, const void* v, const float* la,
                            const float* beta, void* o, int nh, cudaStream_t s, const uint8_t* qs = nullptr,
                            const uint8_t* ks = nullptr, const uint8_t* vs = nullptr) {
    return launch_chained(decode_step_kernel<T, DK, DV, MX>, dim3(nh), dim3(256), s, state, q, k, v, qs, ks, vs, la,
                          beta, static_cast<T*>(o));
}

template <typename T, int DK, int DV>
cudaError_t launch_multi_t(float* state, const void* q, const void* k, const void* v, const float* la,
                           const float* beta, int n, int H, int n_draft, const int32_t* n_accept, void* o,
                           int* status, cudaStream_t s) {
    const T* qq = static_cast<const T*>(q);
    const T* kk = static_cast<const T*>(k);
    const T* vv = static_cast<const T*>(v);
    const dim3 grid(n * H, DV / kSpecSlice), block(spec_threads<DV>());
    // the first drafts' inputs are copied to shared memory 16 bytes at a time when every base is 16-byte
    // aligned (every row and slice offset is a multiple of 16 bytes); otherwise they are loaded per element
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    const bool pre16 = a16(kk) && a16(vv) && a16(la) && (n_accept || a16(qq));
    if (n_accept)
        return launch_chained(decode_multi_kernel<T, DK, DV, false>, grid, block, s, state, qq, kk, vv, la, beta, H,
                              n_draft, n_accept, static_cast<T*>(nullptr), pre16, status);
    return launch_chained(decode_multi_kernel<T, DK, DV, true>, grid, block, s, state, qq, kk, vv, la, beta, H,
                          n_draft, static_cast<const int32_t*>(nullptr), static_cast<T*>(o), pre16, status);
}

}  // namespace

cudaError_t launch_decode(float* state, const void* q, const void* k, const void* v, const float* la,
                          const float* beta, void* o, int nh, int dk, int dv, bool bf16, cudaStream_t s) {
    if (nh == 0) return cudaSuccess;
#define KDA_DECODE_CASE(T, DK, DV) \
    if (dk == DK && dv == DV) return launch_decode_t<T, DK, DV>(state, q, k, v, la, beta, o, nh, s);
    if (bf16) {
        KDA_DECODE_CASE(__nv_bfloat16, 128, 128) KDA_DECODE_CASE(__nv_bfloat16, 128, 64)
        KDA_DECODE_CASE(__nv_bfloat16, 64, 128) KDA_DECODE_CASE(__nv_bfloat16, 64, 64)
    } else {
        KDA_DECODE_CASE(float, 128, 128) KDA_DECODE_CASE(float, 128, 64)
        KDA_DECODE_CASE(float, 64, 128) KDA_DECODE_CASE(float, 64, 64)
    }
#undef KDA_DECODE_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_mx(float* state, const void* q, const uint8_t* qs, const void* k, const uint8_t* ks,
                             const void* v, const uint8_t* vs, const float* la, const float* beta, void* o, int nh,
                             int dk, int dv, cudaStream_t s) {
    if (nh == 0) return cudaSuccess;
#define KDA_DECODE_MX_CASE(DK, DV) \
    if (dk == DK && dv == DV)       \
        return launch_decode_t<__nv_bfloat16, DK, DV, true>(state, q, k, v, la, beta, o, nh, s, qs, ks, vs);
    KDA_DECODE_MX_CASE(128, 128) KDA_DECODE_MX_CASE(128, 64) KDA_DECODE_MX_CASE(64, 128) KDA_DECODE_MX_CASE(64, 64)
#undef KDA_DECODE_MX_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_multi(float* state, const void* q, const void* k, const void* v, const float* la,
                                const float* beta, int n, int H, int n_draft, const int32_t* n_accept, void* o,
                                int dk, int dv, bool bf16, int* status, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
#define KDA_MULTI_CASE(T, DK, DV)  \
    if (dk == DK && dv == DV)      \
        return launch_multi_t<T, DK, DV>(state, q, k, v, la, beta, n, H, n_draft, n_accept, o, status, s);
    if (bf16) {
        KDA_MULTI_CASE(__nv_bfloat16, 128, 128) KDA_MULTI_CASE(__nv_bfloat16, 128, 64)
        KDA_MULTI_CASE(__nv_bfloat16, 64, 128) KDA_MULTI_CASE(__nv_bfloat16, 64, 64)
    } else {
        KDA_MULTI_CASE(float, 128, 128) KDA_MULTI_CASE(float, 128, 64)
        KDA_MULTI_CASE(float, 64, 128) KDA_MULTI_CASE(float, 64, 64)
    }
#undef KDA_MULTI_CASE
    return cudaErrorInvalidValue;
}

}  // namespace kda
