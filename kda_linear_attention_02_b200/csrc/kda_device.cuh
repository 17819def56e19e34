// kda_device.cuh -- device helpers shared by the libkda kernels (sm_100a only).
//
// Hand-written PTX wrappers for the Blackwell pieces the kernels use: mbarriers with bounded waits,
// bulk and tensor TMA copies, and tcgen05 (TMEM allocation, MMA, commit, loads).  Also the
// per-device status word through which kernels report errors instead of trapping.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// ln(0.0067): the per-step log-decay floor (each step keeps >= 0.67 % of the state; orkas.ai
// "Kimi K3 architecture" post, decay-floor section).  fp32 nearest of -5.005647752585217.
constexpr float kLogFloor = -5.0056477f;
constexpr int kChunk = KDA_CHUNK;   // tokens per chunk
constexpr int kTile = KDA_TILE;     // tokens per tile inside a chunk

// Every bounded wait gives up after this many nanoseconds of the global timer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

// Kernels report errors through a pointer to the per-device status word (0 = OK), defined in
// kda_api.cu and passed to every kernel that can fail; the first error recorded wins.
__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for the phase with the given parity.  On timeout records KDA_ERR_TIMEOUT in *status
// (when status is not null) and returns false; the caller then winds down without touching the
// barrier again.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status,
                                          unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > limit_ns) {
            set_status(status, KDA_ERR_TIMEOUT);
            return false;
        }
    }
}

// ---------------------------------------------------------------- async proxy / TMA
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// 1D bulk copy global -> shared, completion on an mbarrier (transaction bytes).
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// 1D bulk copy shared -> global (bulk async-group completion).
__device__ __forceinline__ void bulk_s2g(void* dst, const void* src_smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src_smem)),
                 "r"(bytes)
                 : "memory");
}
// Warm L2 with the line holding p (no data returned; nothing waits on it).
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
// 16 bytes global -> shared by an asynchronous copy (both addresses 16-byte aligned); cp_async_wait_all
// waits for every such copy this thread issued
__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 2D tensor TMA load (no multicast), completion on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void* dst_smem, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst_smem)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}
// 3D tensor TMA load (no multicast), completion on an mbarrier.
__device__ __forceinline__ void tma_load_3d(void* dst_smem, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}
// Loads of data read exactly once: bypass L1 allocation.
__device__ __forceinline__ float2 ld_once_f2(const float* p) {
    float2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.f32 {%0, %1}, [%2];" : "=f"(r.x), "=f"(r.y) : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ld_once_u32(const void* p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.b32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ld_once_u16(const void* p) {
    unsigned short r;
    asm volatile("ld.global.nc.L1::no_allocate.b16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}
// 16-byte global store.
__device__ __forceinline__ void st_global_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
// 3D tensor TMA store shared -> global (bulk async-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int c0, int c1, const void* src_smem) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(smem_u32(src_smem))
                 : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, int c0, int c1, int c2, const void* src_smem) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(src_smem))
                 : "memory");
}
// Named barrier over `count` threads (id 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Arrive at named barrier `id` (of `count` threads) without waiting: writes before it are visible to the
// threads that pass the barrier with named_bar_sync.
__device__ __forceinline__ void named_bar_arrive(int id, int count) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Programmatic dependent launch: a kernel launched with programmatic stream serialization may start
// while the previous kernel of the stream is still finishing; this waits until that kernel has
// completed and its memory is visible (a no-op for an ordinary launch).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
// Allocation: warp-wide.  Writes the TMEM base address to *dst_smem.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 in, fp32 accumulate), one CTA.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// The same with A in tensor memory: row m of A in lane m, K packed two bf16 per 32-bit column (a K = 16
// slice is 8 columns), starting at column address a_tmem.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the mbarrier when all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Waits for this thread's tcgen05.ld and ties the loaded registers to the wait: each value passes
// through an empty volatile asm after it, so no use of a destination register can be scheduled
// before the wait.
template <int N>
__device__ __forceinline__ void tmem_wait_ld_regs(float* v) {
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}

// 32 lanes x 32 bit, 16 consecutive columns: thread t of the warp gets lane (warp quarter base + t).
// 16 consecutive 32-bit columns of this warp's 32 TMEM lanes from registers; tmem_wait_st before the
// stores are relied on (then tcgen05.fence::before_thread_sync and a barrier for another thread's MMA)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        :
        : "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
          "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
          "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
          "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
          "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
          "r"(__float_as_uint(v[15]))
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr));
}

// 16 lanes x 256 bit, twice along the columns: the accumulator fragment of a warp-level m16n8 product for
// two blocks of 8 columns.  Thread t (g = t / 4, q = t % 4) gets, for block b (columns 8 b .. 8 b + 7 from the
// address's column): r[4 b] = (lane g, column 2 q), r[4 b + 1] = (lane g, column 2 q + 1), r[4 b + 2] =
// (lane g + 8, column 2 q), r[4 b + 3] = (lane g + 8, column 2 q + 1), lanes from the address's lane field.
__device__ __forceinline__ void tmem_ld_16x256b_x2(uint32_t taddr, float* r) {
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
                 : "r"(taddr));
}

// Four 8 x 8 matrices of 16-bit elements between shared memory and the fragment layout: lanes 8 j .. 8 j + 7
// give the shared addresses of the eight 16-byte rows of matrix j, and r[j] of thread t holds the two
// elements (row t / 4; columns 2 (t % 4), 2 (t % 4) + 1) of matrix j, the lower column in the low half.
// The .trans forms exchange rows and columns between memory and the fragment.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t saddr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr)
                 : "memory");
}
__device__ __forceinline__ void stsm_x4(uint32_t saddr, const uint32_t (&r)[4]) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(saddr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3])
                 : "memory");
}
__device__ __forceinline__ void stsm_x4_trans(uint32_t saddr, const uint32_t (&r)[4]) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(saddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
}

// Shared-memory matrix descriptor, K-major operand with the 128-byte swizzle: 8-row core groups of
// 8 x 128 B (1024 B, SBO), rows 128 B apart, 16-byte chunks XOR-permuted by (row % 8).  The tile
// base must be 1024-byte aligned; stepping K by 16 bf16 inside the 128-byte row adds 32 B to the
// start address.  Bits: start>>4 [0,14), LBO>>4 [16,30), SBO>>4 [32,46), version 1 at [46,48),
// layout 2 (128B swizzle) at [61,64).
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;              // LBO: unused for swizzled K-major (1 by convention)
    d |= static_cast<uint64_t>((1024u >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;              // descriptor version for sm_100
    d |= static_cast<uint64_t>(2u) << 61;              // SWIZZLE_128B
    return d;
}
// Shared-memory matrix descriptor, MN-major operand with the 128-byte swizzle: each K row holds
// 64 consecutive MN elements (128 B, 16-byte chunks XOR-permuted by (k % 8)); 8 K rows form a
// 1024-byte atom; atoms follow each other along K (SBO = 1024); the next 64 MN elements start
// lbo_bytes further.  Stepping K by 16 adds 2048 B to the start address.
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t saddr, uint32_t lbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((1024u >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}
// Instruction descriptor: kind::f16 with A = B = bf16, D = fp32, shape M x N; A K-major, B K-major
// unless b_mn (then MN-major).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool negate_a = false, bool b_mn = false,
                                                 bool a_mn = false) {
    return (1u << 4)                       // D format: f32
           | (1u << 7)                     // A format: bf16
           | (1u << 10)                    // B format: bf16
           | ((negate_a ? 1u : 0u) << 13)  // negate A
           | ((a_mn ? 1u : 0u) << 15)      // A major-ness
           | ((b_mn ? 1u : 0u) << 16)      // B major-ness
           | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
// Byte offset of element (mn, k) in an MN-major 128B-swizzled tile ([mn/64 blocks of lbo bytes]
// [k/8 atoms of 1024 B][k%8 rows of 128 B]).
__host__ __device__ __forceinline__ uint32_t sw128_mn_offset(int mn, int k, uint32_t lbo_bytes) {
    return static_cast<uint32_t>((mn >> 6) * lbo_bytes + (k >> 3) * 1024 + (k & 7) * 128 +
                                 ((((mn & 63) >> 3) ^ (k & 7)) << 4) + (mn & 7) * 2);
}

// Byte offset of element (row, k) in a K-major 128B-swizzled tile of `rows` rows whose K extent is
// split into 64-element (128-byte) atoms stored one after another ([katom][rows][128 B]).
__host__ __device__ __forceinline__ uint32_t sw128_offset(int row, int k, int rows) {
    const int katom = k >> 6;
    const int kk = k & 63;
    const int chunk = (kk >> 3) ^ (row & 7);
    return static_cast<uint32_t>(katom * rows * 128 + row * 128 + chunk * 16 + (kk & 7) * 2);
}

// ---------------------------------------------------------------- small numeric helpers
__device__ __forceinline__ float floor_log_decay(float la) { return fmaxf(la, kLogFloor); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------- warp-level tf32 MMA for tiny products
// fp32 -> tf32 operand (round to nearest, 10 explicit mantissa bits)
__device__ __forceinline__ uint32_t to_tf32(float f) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(f));
    return r;
}
// d (16 x 8, fp32) += a (16 x 8, row-major) . b (8 x 8).  With g = lane / 4 and c = lane % 4:
// a = {A[g][c], A[g+8][c], A[g][c+4], A[g+8][c+4]}, b = {B[c][g], B[c+4][g]},
// d = {D[g][2c], D[g][2c+1], D[g+8][2c], D[g+8][2c+1]}.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// MXFP8 inputs (OCP Microscaling Formats v1.0).  Two E4M3 codes (the first in the low byte of u) to
// fp32 by the hardware conversion to an f16 pair: every E4M3 value is exact in f16 (|x| <= 448, finest step
// 2^-9), the NaN codes S.1111.111 become NaN, and the widening to fp32 is exact.  The shared scale then
// follows as one power-of-two multiply, exact unless the value leaves the fp32 range.
__device__ __forceinline__ float2 e4m3x2_to_f2(uint32_t u) {
    uint32_t h;
    asm("{\n .reg .b16 c;\n cvt.u16.u32 c, %1;\n cvt.rn.f16x2.e4m3x2 %0, c;\n}" : "=r"(h) : "r"(u));
    return __half22float2(*reinterpret_cast<__half2*>(&h));
}
// E8M0 shared scale -> 2^(e - 127) (code 0 is the fp32 subnormal 2^-127, code 255 is NaN)
__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
    return e == 255u ? __uint_as_float(0x7FC00000u) : __uint_as_float(e ? e << 23 : 0x00400000u);
}
// One MXFP8 element: code c with the shared scale code e of its 32-element block.
__device__ __forceinline__ float mx8_value(uint32_t c, uint32_t e) {
    return e4m3x2_to_f2(c).x * e8m0_to_f32(e);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

}  // namespace kda
