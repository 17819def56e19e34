// kda_compose.cu -- segment composition by prefix scan on one GPU.
//
// Sequence split of the orkas.ai "Kimi K3 architecture" post (section "비용은 서빙 스택에서
// 돌아옵니다"): a plain sum of zero-start states is wrong for KDA because every token applies a
// token-dependent transition to the incoming state; instead each segment is summarised by its
// cumulative transition M_s and its zero-start state Z_s, and a prefix scan recovers every segment's
// start state:  X_0 = init,  X_{s+1} = M_s X_s + Z_s.
//
// The dv columns of X evolve independently, so a CTA owns one (sequence, head, 32-column slice)
// and walks that sequence's segments in order.  Per segment it stages M_s^T in shared memory and
// forms the 128 x 32 product with 4 x 4 register blocking in fp32.
#include "kda_device.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int kComposeCols = 32;

template <int DK, int DV>
__global__ void __launch_bounds__(256)
compose_kernel(const float* __restrict__ M, const float* __restrict__ Z, const int32_t* __restrict__ seg_cu,
               const float* __restrict__ init, int n_seqs, int n_segs, int H, float* __restrict__ starts,
               float* __restrict__ ends, int* status) {
    constexpr int NC = kComposeCols;
    constexpr int MT_LD = DK + 4;            // padded row of M^T (keeps float4 alignment)
    constexpr int TR = DK / 32;              // rows per thread (4 for DK = 128)
    extern __shared__ __align__(16) float smem[];
    float* Mt = smem;                        // [DK][MT_LD]  (M^T: Mt[m][i] = M[i][m])
    float* X = Mt + DK * MT_LD;              // [DK][NC]

    const int seq = blockIdx.x / H;
    const int h = blockIdx.x % H;
    const int c0 = blockIdx.y * NC;
    const int t = threadIdx.x;
    const int tj = t & 7;                    // 4 columns: 4*tj .. 4*tj+3
    const int ti = t >> 3;                   // rows ti*TR .. ti*TR+TR-1 (ti in 0..31)

    const int s0 = seg_cu[seq], s1 = seg_cu[seq + 1];
    if (s0 < 0 || s1 < s0 || s1 > n_segs || (seq == 0 && s0 != 0) || (seq == n_seqs - 1 && s1 != n_segs)) {
        if (t == 0) set_status(status, KDA_ERR_DEVICE_INPUT);
        return;
    }

    for (int e = t; e < DK * NC; e += 256) {
        const int i = e / NC, j = e % NC;
        X[e] = init ? init[((static_cast<size_t>(seq) * H + h) * DK + i) * DV + c0 + j] : 0.f;
    }
    __syncthreads();

    for (int s = s0; s < s1; ++s) {
        const size_t base_s = (static_cast<size_t>(s) * H + h);
        // start state of segment s
        for (int e = t; e < DK * NC; e += 256) {
            const int i = e / NC, j = e % NC;
            starts[(base_s * DK + i) * DV + c0 + j] = X[e];
        }
        // stage M_s^T
        const float* Ms = M + base_s * DK * DK;
        for (int e = t; e < DK * DK; e += 256) {
            const int i = e / DK, m = e % DK;
            Mt[m * MT_LD + i] = Ms[e];
        }
        __syncthreads();
        float acc[TR][4];
        const float* Zs = Z + base_s * DK * DV;
#pragma unroll
        for (int r = 0; r < TR; ++r) {
            const float4 z = *reinterpret_cast<const float4*>(Zs + (ti * TR + r) * DV + c0 + 4 * tj);
            acc[r][0] = z.x; acc[r][1] = z.y; acc[r][2] = z.z; acc[r][3] = z.w;
        }
#pragma unroll 4
        for (int m = 0; m < DK; ++m) {
            const float4 xm = *reinterpret_cast<const float4*>(X + m * NC + 4 * tj);
            float mi[TR];
#pragma unroll
            for (int r = 0; r < TR; ++r) mi[r] = Mt[m * MT_LD + ti * TR + r];
#pragma unroll
            for (int r = 0; r < TR; ++r) {
                acc[r][0] = fmaf(mi[r], xm.x, acc[r][0]);
                acc[r][1] = fmaf(mi[r], xm.y, acc[r][1]);
                acc[r][2] = fmaf(mi[r], xm.z, acc[r][2]);
                acc[r][3] = fmaf(mi[r], xm.w, acc[r][3]);
            }
        }
        __syncthreads();   // all reads of X and Mt done
#pragma unroll
        for (int r = 0; r < TR; ++r)
            *reinterpret_cast<float4*>(X + (ti * TR + r) * NC + 4 * tj) =
                make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
        __syncthreads();
    }
    if (ends) {
        for (int e = t; e < DK * NC; e += 256) {
            const int i = e / NC, j = e % NC;
            ends[((static_cast<size_t>(seq) * H + h) * DK + i) * DV + c0 + j] = X[e];
        }
    }
}

template <int DK, int DV>
static cudaError_t launch_compose_t(const float* M, const float* Z, const int32_t* seg_cu, const float* init,
                                    int n_seqs, int n_segs, int H, float* starts, float* ends, int* status,
                                    cudaStream_t s) {
    const size_t smem = (static_cast<size_t>(DK) * (DK + 4) + static_cast<size_t>(DK) * kComposeCols) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(compose_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(n_seqs * H, DV / kComposeCols);
    compose_kernel<DK, DV><<<grid, 256, smem, s>>>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status);
    return cudaGetLastError();
}

cudaError_t launch_compose(const float* M, const float* Z, const int32_t* seg_cu, const float* init, int n_seqs,
                           int n_segs, int H, int dk, int dv, float* starts, float* ends, int* status,
                           cudaStream_t s) {
    if (n_seqs == 0) return cudaSuccess;
    if (dk == 128 && dv == 128) return launch_compose_t<128, 128>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
    if (dk == 128 && dv == 64) return launch_compose_t<128, 64>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
    if (dk == 64 && dv == 128) return launch_compose_t<64, 128>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
    return launch_compose_t<64, 64>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
}

}  // namespace kda
