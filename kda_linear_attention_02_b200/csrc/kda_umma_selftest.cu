// kda_umma_selftest.cu -- diagnostics of the tcgen05 path the chunk kernels use, no KDA arithmetic:
//  * one bf16 product through the same shared-memory descriptors (128-byte swizzle; A and B each K-major
//    or MN-major), TMEM allocation, commit and TMEM-load path: D[128, n] = A[128, 64] * B[n, 64]^T, with A
//    from shared memory or from tensor memory (row m in lane m, two bf16 per 32-bit column);
//  * the tensor-core rate of a product shape as the kernels issue it (M = 128 x N x K, one CTA per SM,
//    timed with the SM clock): back to back, and one product at a time waited for before the next.
#include "kda_device.cuh"
#include "kda_internal.h"

namespace kda {

__global__ void __launch_bounds__(128) selftest_umma_kernel(const __nv_bfloat16* __restrict__ a,
                                                            const __nv_bfloat16* __restrict__ b,
                                                            float* __restrict__ d, int n, int flags, int* status) {
    const int b_mn = flags & 1, a_tmem = flags & 2, a_mn = flags & 4, m64 = flags & 8;
    extern __shared__ __align__(1024) uint8_t raw[];
    uint8_t* base = raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);   // stays a shared-memory pointer
    uint8_t* sA = base;                 // 128 rows x 128 B
    uint8_t* sB = base + 128 * 128;     // n rows x 128 B
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tbase;
    const int t = threadIdx.x, w = t >> 5, lane = t & 31;

    const uint32_t lbo = 8 * 1024;   // MN-major: 64 K rows = 8 atoms per 64-element MN block
    if (a_mn) {   // two 64-row M blocks, each [64 k][128 B]
        for (int e = t; e < 128 * 64; e += 128) {
            const int r = e >> 6, k = e & 63;
            *reinterpret_cast<__nv_bfloat16*>(sA + sw128_mn_offset(r, k, lbo)) = a[r * 64 + k];
        }
    } else {
        // stage rows into the K-major 128B-swizzled layout: 16-byte chunk c of row r goes to chunk c ^ (r % 8)
        for (int e = t; e < 128 * 8; e += 128) {
            const int r = e >> 3, c = e & 7;
            const uint4 x = reinterpret_cast<const uint4*>(a + r * 64)[c];
            *reinterpret_cast<uint4*>(sA + sw128_offset(r, c * 8, 128)) = x;
        }
    }
    if (b_mn) {
        for (int e = t; e < n * 64; e += 128) {
            const int r = e >> 6, k = e & 63;
            *reinterpret_cast<__nv_bfloat16*>(sB + sw128_mn_offset(r, k, lbo)) = b[r * 64 + k];
        }
    } else {
        for (int e = t; e < n * 8; e += 128) {
            const int r = e >> 3, c = e & 7;
            const uint4 x = reinterpret_cast<const uint4*>(b + r * 64)[c];
            *reinterpret_cast<uint4*>(sB + sw128_offset(r, c * 8, n)) = x;
        }
    }
    fence_proxy_async_smem();
    if (t == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    if (w == 0) {
        tmem_alloc(&tbase, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tbase;
    if (a_tmem) {   // row 32 w + lane of A into TMEM columns [256, 288) of this warp's lanes
        const uint32_t* ar = reinterpret_cast<const uint32_t*>(a + (32 * w + lane) * 64);
        for (int c0 = 0; c0 < 32; c0 += 16) {
            float x[16];
            for (int j = 0; j < 16; ++j) x[j] = __uint_as_float(ar[c0 + j]);
            tmem_st16(tm + (static_cast<uint32_t>(32 * w) << 16) + 256 + c0, x);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (t == 0) {
        const uint32_t idesc = idesc_bf16(m64 ? 64 : 128, n, false, b_mn != 0, a_mn != 0);
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t db = b_mn ? sdesc_mn_sw128(smem_u32(sB) + kk * 2048, lbo)
                                     : sdesc_k_sw128(smem_u32(sB) + kk * 32);
            const uint64_t da = a_mn ? sdesc_mn_sw128(smem_u32(sA) + kk * 2048, lbo)
                                     : sdesc_k_sw128(smem_u32(sA) + kk * 32);
            if (a_tmem) umma_f16_ts(tm, tm + 256 + kk * 8, db, idesc, kk > 0);
            else umma_f16(tm, da, db, idesc, kk > 0);
        }
        umma_commit(&bar);
    }
    __syncwarp();
    const bool ok = mbar_wait(&bar, 0, status);
    tc_fence_after();
    if (ok) {
        for (int c0 = 0; c0 < n; c0 += 16) {
            float r[16];
            tmem_ld16(tm + (static_cast<uint32_t>(32 * w) << 16) + c0, r);
            tmem_wait_ld_regs<16>(r);
            for (int j = 0; j < 16; ++j) d[(32 * w + lane) * n + c0 + j] = r[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tm, 512);
}

// One CTA per SM; thread 0 times `reps` products of shape 128 x n x k (operands zero: only the timing
// matters) issued back to back with one commit at the end, then `reps` products each committed and waited
// for before the next.  cycles[2 * blockIdx.x + {0, 1}] = SM cycles per product in the two modes.
__global__ void __launch_bounds__(128) selftest_mma_rate_kernel(int n, int k, int majors, int reps, float* cycles,
                                                                int* status) {
    const int b_mn = majors & 1, a_mn = majors & 4, m64 = majors & 8;
    extern __shared__ __align__(1024) uint8_t raw[];
    uint8_t* base = raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
    uint8_t* sA = base;                          // K-major [k / 64][128 rows][128 B] or MN-major [2][k][128 B]
    uint8_t* sB = base + (k / 64) * 16384;       // K-major [k / 64][n][128 B] or MN-major [n / 64][k][128 B]
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tbase;
    const int t = threadIdx.x, w = t >> 5;
    const int words = ((k / 64) * 16384 + n * k * 2) / 16;
    for (int e = t; e < words; e += 128) reinterpret_cast<uint4*>(base)[e] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    if (t == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    if (w == 0) {
        tmem_alloc(&tbase, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tbase;
    if (t == 0) {
        const uint32_t idesc = idesc_bf16(m64 ? 64 : 128, n, false, b_mn != 0, a_mn != 0);
        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
        auto product = [&]() {
            for (int ks = 0; ks < k / 16; ++ks) {
                const uint64_t da = a_mn ? sdesc_mn_sw128(a0 + ks * 2048, static_cast<uint32_t>(k) * 128)
                                         : sdesc_k_sw128(a0 + (ks >> 2) * 16384 + (ks & 3) * 32);
                const uint64_t db = b_mn ? sdesc_mn_sw128(b0 + ks * 2048, static_cast<uint32_t>(k) * 128)
                                         : sdesc_k_sw128(b0 + (ks >> 2) * n * 128 + (ks & 3) * 32);
                umma_f16(tm, da, db, idesc, ks > 0);
            }
        };
        uint32_t ph = 0;
        bool ok = true;
        product();                               // warm-up
        umma_commit(&bar);
        ok = ok && mbar_wait(&bar, ph, status);
        ph ^= 1;
        const long long t0 = clock64();
        for (int r = 0; r < reps; ++r) product();
        umma_commit(&bar);
        ok = ok && mbar_wait(&bar, ph, status);
        ph ^= 1;
        const long long t1 = clock64();
        for (int r = 0; r < reps && ok; ++r) {
            product();
            umma_commit(&bar);
            ok = mbar_wait(&bar, ph, status);
            ph ^= 1;
        }
        const long long t2 = clock64();
        cycles[2 * blockIdx.x] = ok ? static_cast<float>(t1 - t0) / reps : -1.f;
        cycles[2 * blockIdx.x + 1] = ok ? static_cast<float>(t2 - t1) / reps : -1.f;
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tm, 256);
}

cudaError_t launch_selftest_mma_rate(int n, int k, int majors, int reps, float* cycles, int grid, int* status,
                                     cudaStream_t s) {
    const int smem = 1024 + (k / 64) * 16384 + n * k * 2;
    cudaError_t e = cudaFuncSetAttribute(selftest_mma_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    selftest_mma_rate_kernel<<<grid, 128, smem, s>>>(n, k, majors, reps, cycles, status);
    return cudaGetLastError();
}

cudaError_t launch_selftest_umma(const void* a, const void* b, float* d, int n, int flags, int* status,
                                 cudaStream_t s) {
    const int smem = 1024 + 128 * 128 + ((n + 63) / 64) * 64 * 128;
    cudaError_t e = cudaFuncSetAttribute(selftest_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    selftest_umma_kernel<<<1, 128, smem, s>>>(static_cast<const __nv_bfloat16*>(a),
                                              static_cast<const __nv_bfloat16*>(b), d, n, flags, status);
    return cudaGetLastError();
}

}  // namespace kda
