// kda_compose.cu -- segment composition by prefix scan on one GPU.
//
// Sequence split of the orkas.ai "Kimi K3 architecture" post (section "비용은 서빙 스택에서
// 돌아옵니다"): a plain sum of zero-start states is wrong for KDA because every token applies a
// token-dependent transition to the incoming state; instead each segment is summarised by its
// cumulative transition M_s and its zero-start state Z_s, and a prefix scan recovers every segment's
// start state:  X_0 = init,  X_{s+1} = M_s X_s + Z_s.
//
// dk = 128 (compose_tc_kernel): one CTA per (sequence, head) walks the sequence's segments in order
// and forms M_s X_s on the tensor cores.  fp32 accuracy comes from splitting every fp32 operand value
// into three bf16 pieces x = x1 + x2 + x3 (x1 = bf16(x), x2 = bf16(x - x1), x3 = bf16(x - x1 - x2): 24
// significant bits) and summing the six products x1 y1 + x1 y2 + x2 y1 + x1 y3 + x3 y1 + x2 y2 in the
// fp32 accumulator; the terms left out are below 2^-24 of |M| |X|.  M_s is a K-major operand (rows i,
// K = m), X_s an MN-major one (K rows m, N = dv columns j), both with the 128-byte swizzle.
// dk = 64 (compose_kernel): the dv columns of X evolve independently, so a CTA owns one (sequence,
// head, 32-column slice) and walks the segments in order, staging M_s^T in shared memory and forming
// the 64 x 32 product with 4 x 4 register blocking in fp32.
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

// three bf16 pieces of x (their sum holds x to 24 significant bits)
__device__ __forceinline__ void split3(float x, float& a, float& b, float& c) {
    a = __bfloat162float(__float2bfloat16_rn(x));
    const float r = x - a;
    b = __bfloat162float(__float2bfloat16_rn(r));
    c = r - b;
}

template <int DV>
struct ComposeTc {
    static constexpr int NT = 256;
    static constexpr uint32_t A_PIECE = 128 * 128 * 2;      // M_s piece: [2 K atoms][128 rows][128 B]
    static constexpr uint32_t B_PIECE = DV * 128 * 2;       // X_s piece: [DV / 64 blocks][128 K rows][128 B]
    static constexpr uint32_t A0 = 0, B0 = 3 * A_PIECE;
    static constexpr uint32_t BYTES = B0 + 3 * B_PIECE;
    static constexpr uint32_t LBO = 128 * 128;             // MN-major: 64 columns x 128 K rows per block
};

template <int DV>
__global__ void __launch_bounds__(256, 1)
compose_tc_kernel(const float* __restrict__ M, const float* __restrict__ Z, const int32_t* __restrict__ seg_cu,
                  const float* __restrict__ init, int n_seqs, int n_segs, int H, float* __restrict__ starts,
                  float* __restrict__ ends, int* status) {
    using C = ComposeTc<DV>;
    constexpr int DK = 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tmem_slot;
    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    const int seq = blockIdx.x / H, h = blockIdx.x % H;
    const int s0 = seg_cu[seq], s1 = seg_cu[seq + 1];
    if (s0 < 0 || s1 < s0 || s1 > n_segs || (seq == 0 && s0 != 0) || (seq == n_seqs - 1 && s1 != n_segs)) {
        if (t == 0) set_status(status, KDA_ERR_DEVICE_INPUT);
        return;
    }
    if (t == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    if (w == 0) {
        tmem_alloc(&tmem_slot, 128);
        tmem_relinquish();
    }
    // X as the MN-major B operand pieces: thread = (row i = t >> 1, half of the DV columns), 8 columns per
    // 16-byte chunk of each piece
    auto put_x_row8 = [&](int i, int j, const float (&x)[8]) {
        float a[8], b[8], c[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) split3(x[e], a[e], b[e], c[e]);
        const uint32_t off = C::B0 + sw128_mn_offset(j, i, C::LBO);
        *reinterpret_cast<uint4*>(sm + off) = make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                                                         pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
        *reinterpret_cast<uint4*>(sm + off + C::B_PIECE) = make_uint4(pack_bf16x2(b[0], b[1]), pack_bf16x2(b[2], b[3]),
                                                                      pack_bf16x2(b[4], b[5]), pack_bf16x2(b[6], b[7]));
        *reinterpret_cast<uint4*>(sm + off + 2 * C::B_PIECE) =
            make_uint4(pack_bf16x2(c[0], c[1]), pack_bf16x2(c[2], c[3]), pack_bf16x2(c[4], c[5]), pack_bf16x2(c[6], c[7]));
    };
    const size_t sh0 = static_cast<size_t>(seq) * H + h;
    {   // X_0 = init (or zero): pieces, and the first segment's start state
        const int i = t >> 1, j0 = (t & 1) * (DV / 2);
        const float* src = init ? init + (sh0 * DK + i) * DV : nullptr;
        float* dst = s1 > s0 ? starts + ((static_cast<size_t>(s0) * H + h) * DK + i) * DV : nullptr;
#pragma unroll
        for (int jj = 0; jj < DV / 2; jj += 8) {
            float x[8];
            const float4 u = src ? *reinterpret_cast<const float4*>(src + j0 + jj) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 v = src ? *reinterpret_cast<const float4*>(src + j0 + jj + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
            x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w; x[4] = v.x; x[5] = v.y; x[6] = v.z; x[7] = v.w;
            if (dst) {
                reinterpret_cast<float4*>(dst + j0 + jj)[0] = u;
                reinterpret_cast<float4*>(dst + j0 + jj)[1] = v;
            }
            put_x_row8(i, j0 + jj, x);
        }
        if (s1 == s0 && ends) {   // no segments: the end state is the initial state
            float* e = ends + (sh0 * DK + i) * DV + j0;
#pragma unroll
            for (int jj = 0; jj < DV / 2; jj += 4)
                *reinterpret_cast<float4*>(e + jj) =
                    src ? *reinterpret_cast<const float4*>(src + j0 + jj) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_slot;
    uint32_t ph = 0;
    for (int s = s0; s < s1; ++s) {
        const size_t bs = static_cast<size_t>(s) * H + h;
        {   // the accumulator starts as Z_s (TMEM stores from the rows' loads): lane quarter w & 3 holds rows
            // 32 (w & 3) .., warp w >> 2 a half of the columns
            const int qw = w & 3, i = 32 * qw + lane, jh = (w >> 2) * (DV / 2);
            const float* zr = Z + (bs * DK + i) * DV + jh;
            if (s + 1 < s1) {   // the next segment's rows of Z into L2 meanwhile
#pragma unroll
                for (int l = 0; l < DV / 2; l += 32) prefetch_l2(Z + ((bs + H) * DK + i) * DV + jh + l);
            }
            tc_fence_after();
#pragma unroll
            for (int jb = 0; jb < DV / 2; jb += 16) {
                float z[16];
#pragma unroll
                for (int e = 0; e < 16; e += 4) {
                    const float4 v4 = *reinterpret_cast<const float4*>(zr + jb + e);
                    z[e] = v4.x; z[e + 1] = v4.y; z[e + 2] = v4.z; z[e + 3] = v4.w;
                }
                tmem_st16(tm + (static_cast<uint32_t>(32 * qw) << 16) + jh + jb, z);
            }
            tmem_wait_st();
            tc_fence_before();
        }
        {   // M_s as three K-major A operand pieces: thread = (row i, 64-column half)
            const int i = t >> 1, m0 = (t & 1) * 64;
            const float* src = M + (bs * DK + i) * DK + m0;
            if (s + 1 < s1) {   // the next segment's rows into L2 meanwhile
                const float* nx = M + ((bs + H) * DK + i) * DK + m0;
                prefetch_l2(nx);
                prefetch_l2(nx + 32);
            }
#pragma unroll
            for (int mm = 0; mm < 64; mm += 8) {
                const float4 u = *reinterpret_cast<const float4*>(src + mm);
                const float4 v = *reinterpret_cast<const float4*>(src + mm + 4);
                const float x[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
                float a[8], b[8], c[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) split3(x[e], a[e], b[e], c[e]);
                const uint32_t off = C::A0 + sw128_offset(i, m0 + mm, 128);
                *reinterpret_cast<uint4*>(sm + off) = make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                                                                 pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
                *reinterpret_cast<uint4*>(sm + off + C::A_PIECE) =
                    make_uint4(pack_bf16x2(b[0], b[1]), pack_bf16x2(b[2], b[3]), pack_bf16x2(b[4], b[5]),
                               pack_bf16x2(b[6], b[7]));
                *reinterpret_cast<uint4*>(sm + off + 2 * C::A_PIECE) =
                    make_uint4(pack_bf16x2(c[0], c[1]), pack_bf16x2(c[2], c[3]), pack_bf16x2(c[4], c[5]),
                               pack_bf16x2(c[6], c[7]));
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        // D = Z_s + sum over the six piece pairs (a, b) of A_a X_b  (M = 128, N = DV, K = 128)
        if (t == 0) {
            tc_fence_after();
            const uint32_t a0 = smem_u32(sm + C::A0), b0 = smem_u32(sm + C::B0);
            const uint32_t idesc = idesc_bf16(128, DV, false, true);
            constexpr int pa[6] = {0, 0, 1, 0, 2, 1}, pb[6] = {0, 1, 0, 2, 0, 1};
#pragma unroll
            for (int p = 0; p < 6; ++p)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_f16(tm, sdesc_k_sw128(a0 + pa[p] * C::A_PIECE + (ks >> 2) * 16384 + (ks & 3) * 32),
                             sdesc_mn_sw128(b0 + pb[p] * C::B_PIECE + ks * 2048, C::LBO), idesc, 1u);
            umma_commit(&bar);
        }
        const bool ok = mbar_wait(&bar, ph, status);
        ph ^= 1;
        if (__syncthreads_or(!ok)) break;
        tc_fence_after();
        {   // X_{s+1} = D: lane quarter w & 3 holds rows 32 (w & 3) .., warp w >> 2 a half of the columns
            const int qw = w & 3, i = 32 * qw + lane, jh = (w >> 2) * (DV / 2);
            float* dst = s + 1 < s1 ? starts + (((bs + H) * DK) + i) * DV : (ends ? ends + (sh0 * DK + i) * DV : nullptr);
#pragma unroll
            for (int jb = 0; jb < DV / 2; jb += 16) {
                float d[16];
                tmem_ld16(tm + (static_cast<uint32_t>(32 * qw) << 16) + jh + jb, d);
                tmem_wait_ld_regs<16>(d);
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    if (dst) *reinterpret_cast<float4*>(dst + jh + jb + e) = make_float4(d[e], d[e + 1], d[e + 2], d[e + 3]);
                if (s + 1 < s1) {   // the next product's B operand
                    float x8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x8[e] = d[e];
                    put_x_row8(i, jh + jb, x8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x8[e] = d[8 + e];
                    put_x_row8(i, jh + jb + 8, x8);
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncthreads();
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tm, 128);
}

template <int DV>
static cudaError_t launch_compose_tc(const float* M, const float* Z, const int32_t* seg_cu, const float* init,
                                     int n_seqs, int n_segs, int H, float* starts, float* ends, int* status,
                                     cudaStream_t s) {
    const int smem = static_cast<int>(ComposeTc<DV>::BYTES) + 1024;
    cudaError_t e = cudaFuncSetAttribute(compose_tc_kernel<DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    compose_tc_kernel<DV><<<n_seqs * H, 256, smem, s>>>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status);
    return cudaGetLastError();
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
    if (dk == 128 && dv == 128) return launch_compose_tc<128>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
    if (dk == 128 && dv == 64) return launch_compose_tc<64>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
    if (dk == 64 && dv == 128) return launch_compose_t<64, 128>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
    return launch_compose_t<64, 64>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
}

}  // namespace kda
