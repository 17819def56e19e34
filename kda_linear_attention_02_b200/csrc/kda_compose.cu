// kda_compose.cu -- segment composition by prefix scan on one GPU.
//
// Sequence split of the orkas.ai "Kimi K3 architecture" post (section "비용은 서빙 스택에서
// 돌아옵니다"): a plain sum of zero-start states is wrong for KDA because every token applies a
// token-dependent transition to the incoming state; instead each segment is summarised by its
// cumulative transition M_s and its zero-start state Z_s, and a prefix scan recovers every segment's
// start state:  X_0 = init,  X_{s+1} = M_s X_s + Z_s.
//
// dk = 128 (compose_ts_kernel): one CTA per (sequence, head) walks the sequence's segments in order
// and forms M_s X_s on the tensor cores.  fp32 accuracy comes from splitting every fp32 operand value
// into three bf16 pieces x = x1 + x2 + x3 (x1 = bf16(x), x2 = bf16(x - x1), x3 = bf16(x - x1 - x2): 24
// significant bits) and summing the six products x1 y1 + x1 y2 + x2 y1 + x1 y3 + x3 y1 + x2 y2 in the
// fp32 accumulator; the terms left out are below 2^-24 of |M| |X|.  M_s's pieces are the A operand in
// tensor memory (row i in lane i, K = m; two buffers, so that M_{s+1} is split while the products of
// segment s run), X_s's the MN-major B operand in shared memory (K rows m, N = dv columns j, 128-byte
// swizzle); Z_s is added to the product in the epilogue.  M and Z arrive by TMA ahead of their use.
// dk = 64 (compose_kernel): the dv columns of X evolve independently, so a CTA owns one (sequence,
// head, 32-column slice) and walks the segments in order, staging M_s^T in shared memory and forming
// the 64 x 32 product with 4 x 4 register blocking in fp32.
#include <cstring>

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

// The three bf16 pieces a = bf16(x), b = bf16(x - a), c = bf16(x - a - b) of a pair of values (their sums
// hold x to 24 significant bits), as packed bf16x2 words (low half = x0): each piece is rounded once and
// its fp32 value read back from the packed word (x - a and x - a - b are exact in fp32).
__device__ __forceinline__ void split3x2(float x0, float x1, uint32_t& pa, uint32_t& pb, uint32_t& pc) {
    pa = pack_bf16x2(x0, x1);
    const float r0 = x0 - __uint_as_float(pa << 16), r1 = x1 - __uint_as_float(pa & 0xFFFF0000u);
    pb = pack_bf16x2(r0, r1);
    pc = pack_bf16x2(r0 - __uint_as_float(pb << 16), r1 - __uint_as_float(pb & 0xFFFF0000u));
}

template <int DV>
struct ComposeTs {
    static constexpr int NT = 256;
    static constexpr uint32_t B_PIECE = DV * 128 * 2;      // X_s piece: [DV / 64 blocks][128 K rows][128 B]
    static constexpr uint32_t B0 = 0;
    // M_s and Z_s staged by TMA as fp32 boxes of [128 rows][32 columns] with the 128-byte swizzle (16 KB each)
    static constexpr uint32_t MS = B0 + 3 * B_PIECE;
    static constexpr uint32_t ZS = MS + 4 * 16384;
    static constexpr uint32_t BYTES = ZS + (DV / 32) * 16384;
    static constexpr uint32_t LBO = 128 * 128;             // MN-major: 64 columns x 128 K rows per block
    // TMEM (512 columns): the accumulator at [0, 128); two buffers of M's three pieces (A operand, row i in
    // lane i, two bf16 of K per column), buffer b's piece p at [TA + 192 b + 64 p, + 64): the pieces of
    // M_{s+1} are formed while the products of segment s read those of M_s
    static constexpr uint32_t TA = 128;
    __host__ __device__ static constexpr uint32_t abuf(int b) { return TA + 192u * static_cast<uint32_t>(b); }
    static_assert(MS % 1024 == 0 && ZS % 1024 == 0, "TMA boxes with the 128-byte swizzle on 1024-byte boundaries");
    static_assert(BYTES + 1024 <= 232448, "one CTA per SM");
};

template <int DV>
__global__ void __launch_bounds__(256, 1)
compose_ts_kernel(const __grid_constant__ CUtensorMap map_m, const __grid_constant__ CUtensorMap map_z,
                  const __grid_constant__ CUtensorMap map_s, const __grid_constant__ CUtensorMap map_e,
                  const int32_t* __restrict__ seg_cu, const float* __restrict__ init, int n_seqs, int n_segs, int H,
                  float* __restrict__ starts, float* __restrict__ ends, int* status) {
    using C = ComposeTs<DV>;
    constexpr int DK = 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_m, bar_z, bar_mma;
    __shared__ uint32_t tmem_slot;
    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    const int seq = blockIdx.x / H, h = blockIdx.x % H;
    const int s0 = seg_cu[seq];
    int s1 = seg_cu[seq + 1];
    if (s0 < 0 || s1 < s0 || s1 > n_segs || (seq == 0 && s0 != 0) || (seq == n_seqs - 1 && s1 != n_segs)) {
        if (t == 0) set_status(status, KDA_ERR_DEVICE_INPUT);
        return;
    }
    if (t == 0) {
        mbar_init(&bar_m, 1);
        mbar_init(&bar_z, 1);
        mbar_init(&bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&map_m);
        prefetch_tmap(&map_z);
        prefetch_tmap(&map_s);
        if (ends) prefetch_tmap(&map_e);
    }
    if (w == 0) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    __syncthreads();   // the barriers are initialised before the first load completes on one
    // M_s of this head into MS (one phase of bar_m; thread 0) and Z_s into ZS (one phase of bar_z; thread 32,
    // which also stores each X_{s+1} from ZS and so knows when ZS is free again)
    bool m_pending = false, z_pending = false;
    auto issue_m = [&](int s) {
        const int row = (s * H + h) * DK;
        mbar_arrive_expect_tx(&bar_m, 4 * 16384);
#pragma unroll
        for (int b = 0; b < 4; ++b) tma_load_2d(sm + C::MS + b * 16384, &map_m, 32 * b, row, &bar_m);
        m_pending = true;
    };
    auto issue_z = [&](int s) {
        const int row = (s * H + h) * DK;
        mbar_arrive_expect_tx(&bar_z, (DV / 32) * 16384);
#pragma unroll
        for (int b = 0; b < DV / 32; ++b) tma_load_2d(sm + C::ZS + b * 16384, &map_z, 32 * b, row, &bar_z);
        z_pending = true;
    };
    if (t == 0 && s1 > s0) issue_m(s0);
    if (t == 32 && s1 > s0) issue_z(s0);
    // X as the MN-major B operand pieces, 8 columns per 16-byte chunk of each piece
    auto put_x_row8 = [&](int i, int j, const float (&x)[8]) {
        uint32_t a[4], b[4], c[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split3x2(x[2 * e], x[2 * e + 1], a[e], b[e], c[e]);
        const uint32_t off = C::B0 + sw128_mn_offset(j, i, C::LBO);
        *reinterpret_cast<uint4*>(sm + off) = make_uint4(a[0], a[1], a[2], a[3]);
        *reinterpret_cast<uint4*>(sm + off + C::B_PIECE) = make_uint4(b[0], b[1], b[2], b[3]);
        *reinterpret_cast<uint4*>(sm + off + 2 * C::B_PIECE) = make_uint4(c[0], c[1], c[2], c[3]);
    };
    const size_t sh0 = static_cast<size_t>(seq) * H + h;
    {   // X_0 = init (or zero): pieces, and the first segment's start state; thread = (row i = t >> 1, half)
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
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_slot;
    // TMEM lane quarter w & 3 holds rows 32 (w & 3) ..; warp w >> 2 takes a half of the columns
    const int qw = w & 3, hh = w >> 2, i = 32 * qw + lane;
    const uint32_t lane_base = tm + (static_cast<uint32_t>(32 * qw) << 16);
    uint32_t ph_m = 0, ph_z = 0, ph_mma = 0;
    // row i of M (in MS), columns [64 hh, 64 hh + 64): its three bf16 pieces into TMEM buffer b, 32 columns of
    // M per box
    auto split_m = [&](int b) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint8_t* rowp = sm + C::MS + (2 * hh + q) * 16384 + i * 128;
            float x[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 v = *reinterpret_cast<const float4*>(rowp + ((c ^ (i & 7)) << 4));
                x[4 * c] = v.x; x[4 * c + 1] = v.y; x[4 * c + 2] = v.z; x[4 * c + 3] = v.w;
            }
            float p0[16], p1[16], p2[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                uint32_t a, b, c;
                split3x2(x[2 * e], x[2 * e + 1], a, b, c);
                p0[e] = __uint_as_float(a);
                p1[e] = __uint_as_float(b);
                p2[e] = __uint_as_float(c);
            }
            const uint32_t col = C::abuf(b) + 32 * hh + 16 * q;
            tmem_st16(lane_base + col, p0);
            tmem_st16(lane_base + col + 64, p1);
            tmem_st16(lane_base + col + 128, p2);
        }
    };
    // the pieces of the first segment's M
    bool ok = true;
    if (s1 > s0) {
        ok = mbar_wait(&bar_m, ph_m, status);
        ph_m ^= 1;
        if (t == 0) m_pending = false;
        if (ok) split_m(0);
        tmem_wait_st();
        tc_fence_before();
        fence_proxy_async_smem();   // MS has been read
    }
    if (__syncthreads_or(!ok)) s1 = s0;   // nothing more to do (the status word says why)
    if (t == 0 && s0 + 1 < s1) issue_m(s0 + 1);
    for (int s = s0; s < s1; ++s) {
        const size_t bs = static_cast<size_t>(s) * H + h;
        const int buf = (s - s0) & 1;
        // D = sum over the six piece pairs (a, b) of A_a X_b  (M = 128, N = DV, K = 128), from zero
        if (t == 0) {
            tc_fence_after();
            const uint32_t b0 = smem_u32(sm + C::B0);
            const uint32_t idesc = idesc_bf16(128, DV, false, true);
            constexpr int pa[6] = {0, 0, 1, 0, 2, 1}, pb[6] = {0, 1, 0, 2, 0, 1};
#pragma unroll
            for (int p = 0; p < 6; ++p)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_f16_ts(tm, tm + C::abuf(buf) + 64 * pa[p] + 8 * ks,
                                sdesc_mn_sw128(b0 + pb[p] * C::B_PIECE + ks * 2048, C::LBO), idesc, p > 0 || ks > 0);
            umma_commit(&bar_mma);
        }
        // meanwhile the next segment's M becomes the other buffer's pieces
        bool has_next = s + 1 < s1;
        ok = true;
        if (has_next) {
            ok = mbar_wait(&bar_m, ph_m, status);
            ph_m ^= 1;
            if (t == 0) m_pending = false;
            if (ok) split_m(buf ^ 1);
            fence_proxy_async_smem();   // MS has been read
        }
        ok = mbar_wait(&bar_mma, ph_mma, status) && ok;
        ph_mma ^= 1;
        ok = mbar_wait(&bar_z, ph_z, status) && ok;
        ph_z ^= 1;
        if (t == 32) z_pending = false;
        if (__syncthreads_or(!ok)) break;
        if (t == 0 && s + 2 < s1) issue_m(s + 2);
        tc_fence_after();
        {   // X_{s+1} = D + Z_s, written over Z_s in ZS (each thread rewrites the values it read) for the tensor
            // store, and the next product's B operand
            const int jh = hh * (DV / 2);
#pragma unroll
            for (int jb = 0; jb < DV / 2; jb += 16) {
                float d[16];
                tmem_ld16(lane_base + jh + jb, d);
                // Z_s row i, columns jh + jb .. + 16: box (jh + jb) / 32, 16-byte chunks from (jb % 32) / 4
                uint8_t* zrow = sm + C::ZS + ((jh + jb) >> 5) * 16384 + i * 128;
                float z[16];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int ch = ((jb & 31) >> 2) + c;
                    const float4 v = *reinterpret_cast<const float4*>(zrow + ((ch ^ (i & 7)) << 4));
                    z[4 * c] = v.x; z[4 * c + 1] = v.y; z[4 * c + 2] = v.z; z[4 * c + 3] = v.w;
                }
                tmem_wait_ld_regs<16>(d);
#pragma unroll
                for (int e = 0; e < 16; ++e) d[e] += z[e];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int ch = ((jb & 31) >> 2) + c;
                    *reinterpret_cast<float4*>(zrow + ((ch ^ (i & 7)) << 4)) =
                        make_float4(d[4 * c], d[4 * c + 1], d[4 * c + 2], d[4 * c + 3]);
                }
                if (has_next) {
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
        tmem_wait_st();   // the next buffer's pieces
        tc_fence_before();
        fence_proxy_async_smem();   // the B pieces for the next products; X_{s+1} in ZS for the tensor store
        __syncthreads();
        if (t == 32) {   // X_{s+1} out (the next start state, or the end state), then the next Z into ZS
            const CUtensorMap* mo = has_next ? &map_s : (ends ? &map_e : nullptr);
            const int row = static_cast<int>((has_next ? bs + H : sh0) * DK);
            if (mo) {
#pragma unroll
                for (int b = 0; b < DV / 32; ++b) tma_store_2d(mo, 32 * b, row, sm + C::ZS + b * 16384);
                bulk_commit();
                bulk_wait_read0();
            }
            if (has_next) issue_z(s + 1);
        }
    }
    if (t == 0 && m_pending) mbar_wait(&bar_m, ph_m, nullptr);   // never leave a TMA write in flight
    if (t == 32) {
        if (z_pending) mbar_wait(&bar_z, ph_z, nullptr);
        bulk_wait0();   // nor a store
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tm, 512);
}

// 2D map over a row-major fp32 matrix [rows][cols]: boxes of 32 columns x 128 rows with the 128-byte swizzle
static bool make_map_f32_rows(CUtensorMap* m, const float* base, int cols, long long rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * sizeof(float)};
    const cuuint32_t box[2] = {32u, 128u};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DV>
static cudaError_t launch_compose_ts(const float* M, const float* Z, const int32_t* seg_cu, const float* init,
                                     int n_seqs, int n_segs, int H, float* starts, float* ends, int* status,
                                     cudaStream_t s) {
    CUtensorMap mm, mz, ms, me;
    memset(&mm, 0, sizeof(mm));
    memset(&mz, 0, sizeof(mz));
    memset(&ms, 0, sizeof(ms));
    memset(&me, 0, sizeof(me));
    const long long rows = static_cast<long long>(n_segs) * H * 128, erows = static_cast<long long>(n_seqs) * H * 128;
    if (rows > 0x7fffffffLL || erows > 0x7fffffffLL) return cudaErrorInvalidValue;   // TMA coordinates are 32-bit
    if (rows > 0 && (!make_map_f32_rows(&mm, M, 128, rows) || !make_map_f32_rows(&mz, Z, DV, rows) ||
                     !make_map_f32_rows(&ms, starts, DV, rows)))
        return cudaErrorInvalidValue;
    if (ends && !make_map_f32_rows(&me, ends, DV, erows)) return cudaErrorInvalidValue;
    const int smem = static_cast<int>(ComposeTs<DV>::BYTES) + 1024;
    cudaError_t e = cudaFuncSetAttribute(compose_ts_kernel<DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    compose_ts_kernel<DV><<<n_seqs * H, 256, smem, s>>>(mm, mz, ms, me, seg_cu, init, n_seqs, n_segs, H, starts, ends,
                                                        status);
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
    if (dk == 128 && dv == 128) return launch_compose_ts<128>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
    if (dk == 128 && dv == 64) return launch_compose_ts<64>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
    if (dk == 64 && dv == 128) return launch_compose_t<64, 128>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
    return launch_compose_t<64, 64>(M, Z, seg_cu, init, n_seqs, n_segs, H, starts, ends, status, s);
}

}  // namespace kda
