// kda_decode.cu -- one recurrent KDA step (decode), state updated in place.
//
// The fixed-size state of the llm-wiki "Kimi K3" chapter (section 1: S updated per token, the query
// multiplied into S, O(1) memory) with the per-channel decay of section "GatedDeltaNet과 KDA의 차이"
// and the 0.67 % retention floor of the orkas.ai "Kimi K3 architecture" post (decay-floor section):
//
//   a = exp(max(log_alpha, ln 0.0067));  p = (Diag(a) S)^T k;  u = beta (v - p);
//   S <- Diag(a) S + k u^T;              o = S^T q = (Diag(a) S)^T q + u (k . q)
//
// HBM-bound (about 1.75 flop/byte): the kernel streams each (sequence, head) state once in and once
// out with 128-bit loads/stores, keeps it in registers between the column reduction and the rank-1
// write, and reduces the two column sums (against a*k and a*q) over warps through shared memory.
#include "kda_device.cuh"
#include "kda_internal.h"

namespace kda {

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256, 2)
decode_step_kernel(float* __restrict__ state, const T* __restrict__ q, const T* __restrict__ k,
                   const T* __restrict__ v, const float* __restrict__ log_alpha,
                   const float* __restrict__ beta, T* __restrict__ o) {
    constexpr int CG = DV / 4;     // float4 column groups
    constexpr int RG = 256 / CG;   // row groups
    constexpr int RPT = DK / RG;   // rows per thread
    static_assert(RG * CG == 256 && RPT * RG == DK, "tiling");
    const int head = blockIdx.x;   // sequence * H + h
    const int t = threadIdx.x;
    const int cg = t % CG;
    const int rg = t / CG;

    __shared__ float s_a[DK], s_k[DK], s_q[DK], s_u[DV];
    __shared__ float4 s_red[2][RG][CG];
    __shared__ float s_kq;

    float4* S = reinterpret_cast<float4*>(state + static_cast<size_t>(head) * DK * DV);
    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) s[r] = __ldcs(S + (rg + r * RG) * CG + cg);

    for (int i = t; i < DK; i += 256) {
        s_a[i] = __expf(floor_log_decay(log_alpha[static_cast<size_t>(head) * DK + i]));
        s_k[i] = to_f32(k[static_cast<size_t>(head) * DK + i]);
        s_q[i] = to_f32(q[static_cast<size_t>(head) * DK + i]);
    }
    __syncthreads();

    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg + r * RG;
        const float ak = s_a[i] * s_k[i], aq = s_a[i] * s_q[i];
        pk.x = fmaf(ak, s[r].x, pk.x); pk.y = fmaf(ak, s[r].y, pk.y);
        pk.z = fmaf(ak, s[r].z, pk.z); pk.w = fmaf(ak, s[r].w, pk.w);
        pq.x = fmaf(aq, s[r].x, pq.x); pq.y = fmaf(aq, s[r].y, pq.y);
        pq.z = fmaf(aq, s[r].z, pq.z); pq.w = fmaf(aq, s[r].w, pq.w);
    }
    s_red[0][rg][cg] = pk;
    s_red[1][rg][cg] = pq;
    if (t < 32) {
        float kq = 0.f;
        for (int i = t; i < DK; i += 32) kq = fmaf(s_k[i], s_q[i], kq);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (t == 0) s_kq = kq;
    }
    __syncthreads();

    if (t < DV) {
        const int j = t;
        const float* red0 = reinterpret_cast<const float*>(s_red[0]);
        const float* red1 = reinterpret_cast<const float*>(s_red[1]);
        float p = 0.f, pqj = 0.f;
#pragma unroll
        for (int g = 0; g < RG; ++g) {
            p += red0[g * DV + j];
            pqj += red1[g * DV + j];
        }
        const float vj = to_f32(v[static_cast<size_t>(head) * DV + j]);
        const float u = beta[head] * (vj - p);
        s_u[j] = u;
        o[static_cast<size_t>(head) * DV + j] = from_f32<T>(fmaf(u, s_kq, pqj));
    }
    __syncthreads();

    const float4 u4 = reinterpret_cast<const float4*>(s_u)[cg];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg + r * RG;
        const float a = s_a[i], kk = s_k[i];
        float4 x;
        x.x = fmaf(a, s[r].x, kk * u4.x);
        x.y = fmaf(a, s[r].y, kk * u4.y);
        x.z = fmaf(a, s[r].z, kk * u4.z);
        x.w = fmaf(a, s[r].w, kk * u4.w);
        __stcs(S + i * CG + cg, x);
    }
}

template <typename T, int DK, int DV>
static cudaError_t launch_decode_t(float* state, const void* q, const void* k, const void* v, const float* la,
                                   const float* beta, void* o, int nh, cudaStream_t s) {
    decode_step_kernel<T, DK, DV><<<nh, 256, 0, s>>>(state, static_cast<const T*>(q), static_cast<const T*>(k),
                                                    static_cast<const T*>(v), la, beta, static_cast<T*>(o));
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_decode_dt(float* state, const void* q, const void* k, const void* v, const float* la,
                                    const float* beta, void* o, int nh, int dk, int dv, cudaStream_t s) {
    if (dk == 128 && dv == 128) return launch_decode_t<T, 128, 128>(state, q, k, v, la, beta, o, nh, s);
    if (dk == 128 && dv == 64) return launch_decode_t<T, 128, 64>(state, q, k, v, la, beta, o, nh, s);
    if (dk == 64 && dv == 128) return launch_decode_t<T, 64, 128>(state, q, k, v, la, beta, o, nh, s);
    return launch_decode_t<T, 64, 64>(state, q, k, v, la, beta, o, nh, s);
}

cudaError_t launch_decode(float* state, const void* q, const void* k, const void* v, const float* la,
                          const float* beta, void* o, int nh, int dk, int dv, bool bf16, cudaStream_t s) {
    if (nh == 0) return cudaSuccess;
    return bf16 ? launch_decode_dt<__nv_bfloat16>(state, q, k, v, la, beta, o, nh, dk, dv, s)
                : launch_decode_dt<float>(state, q, k, v, la, beta, o, nh, dk, dv, s);
}

}  // namespace kda
