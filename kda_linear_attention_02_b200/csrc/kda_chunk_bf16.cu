// kda_chunk_bf16.cu -- chunked KDA forward for bf16 inputs on the sm_100a tensor cores (tcgen05).
//
// The chunk algebra (per chunk of C = 64 tokens, positions r; lambda = max(log_alpha, ln 0.0067),
// g = chunk-local inclusive cumsum of lambda, gamma = exp(g)):
//   A[r,s]   = beta_r sum_c k_rc k_sc exp(g_rc - g_sc)   (s < r),     Aqk[r,s] = sum_c q_rc k_sc exp(..)  (s <= r)
//   X = (I + A)^-1 (blocked forward substitution over 16 x 16 tiles)
//   W = X diag(beta) (K * gamma),  U = X diag(beta) V
// and across chunks, with the fp32 state S:
//   U' = U - W S,   O = (Q * gamma) S + Aqk U',   S <- Diag(gamma_C) S + (K * exp(g_C - g))^T U'.
// The inter-chunk step has two dependent products ([-W; Q gamma] S, then Kdec^T U'); the output's
// Aqk U' is a third product beside Kdec^T U', off the chunk-to-chunk critical path.
//
// Decay floor (orkas.ai "Kimi K3 architecture" post, section "GPU 코드 경로 하나를 없앤 하한"): with
// lambda >= ln 0.0067 the cumulative log-decay of a 16-token tile lies in [-80.09, 0], so with the
// tile anchor b_t (g just before tile t) every factor exp(g_r - b_t) <= 1 and exp(b_t - g_s) <= e^80.09
// < 3.39e38 fits bf16.  Diagonal 16 x 16 tiles therefore go through the same dense bf16 tensor-core
// product as every other tile; nothing is computed per position pair in log space.  With row r in
// tile t the key-side operand of tile t is
//   s in tile t:          k_s exp(b_t - g_s)                          (<= e^80.09)
//   s in tile j < t:      k_s exp(b_{j+1} - g_s) exp(b_t - b_{j+1})   (both <= 1)
// and the row side is k_r exp(g_r - b_t) or q_r exp(g_r - b_t) (<= 1).  Entries with s > r are
// finite (|.| <= 128 e^80.09 < fp32 max) and are dropped after the product.
//
// Kernels:
//  prep_bf16_kernel   persistent, two CTAs per SM, one (chunk, head) item at a time per CTA, a window's
//                     chunks taken last to first: TMA tensor loads of the raw tiles (prefetched one item
//                     ahead), SIMT exponentials and operand construction, tcgen05 products for A/Aqk
//                     (4 anchored variants) and for X diag(beta) (-K gamma | V) (which yields -W and U),
//                     X by forward substitution of the four 16 x 16 diagonal blocks and two merge levels
//                     on warp-level tf32 MMAs (the first two per TMEM lane quarter), and bulk TMA stores
//                     of the MMA-ready packet.
//  state_bf16_kernel  one CTA per (sequence, head, dv-slice), warp-specialised: a producer warp
//                     streams packets through a shared-memory ring with bulk TMA, one thread issues
//                     the tcgen05 products per chunk ([-W; Q gamma] S into a double-buffered
//                     accumulator, then Kdec^T U' and Aqk U'; all three transposed on 128-column
//                     slices), 8 or 16 epilogue warps hold the fp32 state in registers and feed bf16
//                     copies of S and U' back as the next operands (S^T through tensor memory on
//                     128-column slices).
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "kda_chunk_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kDK = 128;

// 1024-byte aligned base inside a dynamic shared-memory array.  Offsetting the array pointer itself
// (instead of rounding an integer) keeps the shared address space visible to the compiler, so the
// accesses through it stay shared-memory loads and stores.
__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return p + ((1024u - (smem_u32(p) & 1023u)) & 1023u);
}
__device__ __forceinline__ void st_b32(uint8_t* p, uint32_t v) { *reinterpret_cast<uint32_t*>(p) = v; }
__device__ __forceinline__ float2 bf2_to_f2(uint32_t u) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(h);
}
__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
    const float2 a = bf2_to_f2(u.x), b = bf2_to_f2(u.y), c = bf2_to_f2(u.z), d = bf2_to_f2(u.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}
__device__ __forceinline__ uint32_t pack2(float2 f) { return pack_bf16x2(f.x, f.y); }
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }
constexpr float kLog2e = 1.4426950408889634f;
// 2^x by the ex2.approx instruction in its flush-to-zero form (the form without flushing adds instructions
// to handle subnormals); e^x is taken as 2^(x log2 e), with the scaling done two lanes at a time where it can.
// The in-tile factors pass log-decays inside one 16-token tile, |x| <= 16 |ln 0.0067| log2 e < 116, so
// neither argument nor result is ever subnormal there.  The anchors' factors (exp_ftz) span up to a whole
// chunk and can underflow: a result below 2^-126 becomes 0 instead of a subnormal, which is the deep-underflow
// limit of a decay product (the values it replaces are below 1.2e-38).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float exp_ftz(float x) { return ex2_approx(x * kLog2e); }
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}

// ------------------------------------------------------------------------------------------------
// Packet: everything the inter-chunk pass needs for one (chunk, head), laid out exactly as its
// shared-memory stage so that it moves with plain bulk copies.
template <int DV>
struct Pk {
    // [-W; Q gamma]: 128 x 128 bf16, K-major, 128B swizzle, 2 K atoms of [128 rows][128 B] (16-byte
    // chunks ^ (row % 8)): rows 0..63 -W, rows 64..127 Q gamma
    static constexpr uint32_t AW = 0;
    static constexpr uint32_t KD = 32768;             // Kdec^T: 128 x 64 bf16, K-major, 128B swizzle
    // Aqk (inclusive lower, zero above): 64 x 64 bf16, K-major, 128B swizzle; it follows Kdec^T, so that the
    // 128-row operand starting 64 rows into Kdec^T has Aqk as its rows 64..127
    static constexpr uint32_t AQ = 49152;
    // U per 64-column atom: [DV/64][64 tokens][128 B], 16-byte chunks ^ (token % 8) -- the MN-major
    // 128B-swizzle B operand of the state pass's copy product, and the layout of the O tensor store
    static constexpr uint32_t U = 57344;
    static constexpr uint32_t G = U + DV * 128;       // gamma_C: [128] fp32
    static constexpr uint32_t BYTES = ((G + 512 + 1023) / 1024) * 1024;
};

// ------------------------------------------------------------------------------------------------
// prep kernel: two CTAs share an SM, so one (chunk, head) item's working set fits in about 110 KB of
// shared memory and 256 TMEM columns; while one CTA waits on a tensor-core product, a barrier or its
// loads, the other computes.  Shared memory (bytes from a 1024-aligned base), reused phase by phase:
//   OPB   column pass, per 64-channel half: the row side [K e^(g-b); Q e^(g-b)] (128 x 64 bf16) at +0 and
//         the key side (4 anchored variants stacked into 160 rows, 160 x 64 bf16) at +16384, K-major with
//         the 128B swizzle (the operands of one K half of product A);
//         solve: A (fp32, pitch LDM) at +0 and X (fp32, pitch LDX) at +17408;
//         then [X; X] diag(beta) (bf16, product B's A operand: rows 64..127 repeat rows 0..63) at +0;
//         epilogue: the packet's -W (two 64-column atoms of 64 rows) at +0, U at +16384
//   QG    Q gamma in the packet's layout, [2 atoms][64 tokens][128 B] bf16 (rows 64..127 of [-W; Q gamma])
//   KG    -(K gamma)^T [128 ch][64 tokens] bf16, K-major (product B's B operand, K part)
//   VOP   V [DV/64][64 tokens][128 B] bf16, MN-major with the 128B swizzle (product B's B operand, V
//         part): a TMA tile for bf16 inputs, written by the column pass for MXFP8 inputs
//   IAQ   MXFP8 inputs: the staged q and k code half-tiles at +0; Aqk (64 x 64 bf16, the packet's layout) at +8192
//   MISC  beta[64]; then the tile half-totals [8][64] fp32 (column pass) or the merge scratch (solve)
//   SCF   MXFP8 inputs only: the shared scales as fp32, [q, k, v][64 tokens][4 blocks]
// TMEM (256 columns): product A at [0, 160); then product B: the K part at [0, 128), the V part at
// [128, 128 + DV).
namespace ps {
constexpr uint32_t OPB = 0;
constexpr uint32_t BVAR = 16384;                 // key side, inside OPB
constexpr uint32_t AM = 0, XF = 17408;           // solve, inside OPB
constexpr uint32_t QG = 36864;
constexpr uint32_t KG = QG + 16384;
constexpr uint32_t VOP = KG + 16384;
constexpr uint32_t IAQ = VOP + 16384;
constexpr uint32_t MISC = IAQ + 16384;           // beta[64] fp32
constexpr uint32_t TOT = MISC + 256;             // [8][64] fp32 (column pass) | [32][LDTT] fp32 (solve)
constexpr uint32_t BYTES = TOT + 5120;
constexpr uint32_t SCF = BYTES;                  // MXFP8 inputs only
constexpr uint32_t BYTES_MX = SCF + 3 * 64 * 16;
constexpr int LDM = 68;              // fp32 row pitch of AM (float4-aligned rows; 4 rows apart = 16 banks)
constexpr int LDX = 73;              // fp32 row pitch of X (odd: column reads of X^T spread over the banks)
constexpr int LDTT = 40;             // fp32 row pitch of the product scratch (8 banks per row: B fragments clash-free)
static_assert(AM + 64 * LDM * 4 <= XF && XF + 64 * LDX * 4 <= QG, "solve scratch inside the operand buffer");
static_assert(32 * LDTT * 4 <= 5120 && 8 * 64 * 4 <= 5120, "column-pass totals and merge scratch share MISC");
constexpr int NT = 256;              // threads per CTA
// two CTAs per SM: (228 KB - 2 x 1 KB reserved) / 2 per CTA, with the 1024-byte alignment slack
static_assert(BYTES_MX + 1024 + 128 <= 115712, "two CTAs per SM");
}  // namespace ps

// MX: q, k, v arrive as MXFP8 (E4M3 codes with one E8M0 scale per 32 channels of a (token, head) row;
// q_scale/k_scale [T, H, 4] and v_scale [T, H, DV / 32] bytes) and are decoded exactly in the column pass;
// everything after it is the bf16 path unchanged.
template <int DV, bool MX>
__global__ void __launch_bounds__(256, 2)
prep_bf16_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_l,
                 const uint8_t* __restrict__ qg, const uint8_t* __restrict__ kg, const uint8_t* __restrict__ vg,
                 const float* __restrict__ lag, const float* __restrict__ beta, const uint8_t* __restrict__ q_scale,
                 const uint8_t* __restrict__ k_scale, const uint8_t* __restrict__ v_scale,
                 const int2* __restrict__ chunk_tab, int H, long long n_items, uint8_t* __restrict__ packets,
                 int* status) {
    using P = Pk<DV>;
    constexpr int NT = ps::NT;
    constexpr int LDM = ps::LDM;
    constexpr int LDX = ps::LDX;
    constexpr int LDTT = ps::LDTT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    __shared__ __align__(8) uint64_t bar_in, bar_mma;
    __shared__ uint32_t tmem_slot;
    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    float* bet = reinterpret_cast<float*>(sm + ps::MISC);
    float* tot = reinterpret_cast<float*>(sm + ps::TOT);   // [8 half tiles][64 channels of the current half]
    // AM holds the strictly lower A = beta_r (K e^g)_r . (K e^-g)_s in two forms that never overlap: the
    // off-diagonal 16 x 16 blocks row-major (AM[r][s], tile(s) < tile(r)), and each diagonal block
    // transposed into its upper triangle (AM[s][r] for s < r in the same tile)
    float* AM = reinterpret_cast<float*>(sm + ps::AM);
    float* XF = reinterpret_cast<float*>(sm + ps::XF);    // X = (I + A)^-1, fp32, pitch LDX
    float* TT = reinterpret_cast<float*>(sm + ps::TOT);   // T = A_10 X_00 of a level-1 merge, pitch LDTT
    float* TS = AM;                                       // T of the level-2 merge, pitch LDTT (rows 0..31 of A)

    if (t == 0) {
        mbar_init(&bar_in, 1);
        mbar_init(&bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&map_q); prefetch_tmap(&map_k); prefetch_tmap(&map_v); prefetch_tmap(&map_l);
    }
    if (w == 0) {
        tmem_alloc(&tmem_slot, 256);   // two CTAs per SM: half of the SM's TMEM each
        tmem_relinquish();
    }
    // Aqk starts at zero: every item rewrites only the columns of its row tile's variant (the entries past
    // them are always zero)
    for (int e = t; e < 64 * 8; e += NT)
        *reinterpret_cast<uint4*>(sm + ps::IAQ + 8192 + 16 * e) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_slot;
    uint32_t ph_in = 0, ph_mma = 0;
    bool in_pending = false;   // a TMA load into VOP is in flight (meaningful in thread 0 only)

    // The k and q tiles of each 64-channel half of an item are staged by TMA (thread 0 issues; each load
    // completes one phase of bar_in).  bf16: VOP takes, in turn, the k and q tiles of the first half
    // ([64 tokens][128 B] each), those of the second half, and finally V as product B's MN-major operand.
    // MXFP8: the code tiles ([64 tokens][64 B] each) go to IAQ + 0, the next item's first half as soon as
    // this item's second half has been read (VOP holds the V the column pass decodes).
    uint8_t* const kq_stage = sm + (MX ? ps::IAQ : ps::VOP);
    constexpr uint32_t kKQ = MX ? 4096 : 8192;   // bytes of one half-tile
    auto issue_kq = [&](long long tok0, int hh, int hf) {
        mbar_arrive_expect_tx(&bar_in, 2 * kKQ);
        tma_load_3d(kq_stage, &map_k, 64 * hf, hh, static_cast<int>(tok0), &bar_in);
        tma_load_3d(kq_stage + kKQ, &map_q, 64 * hf, hh, static_cast<int>(tok0), &bar_in);
        in_pending = true;
    };
    auto issue_v = [&](long long tok0, int hh) {
        if constexpr (!MX) {
            mbar_arrive_expect_tx(&bar_in, DV * 128);
#pragma unroll
            for (int b = 0; b < DV / 64; ++b)
                tma_load_3d(sm + ps::VOP + b * 8192, &map_v, 64 * b, hh, static_cast<int>(tok0), &bar_in);
            in_pending = true;
        }
    };
    // bounded wait for the staging load issued last (all threads)
    auto wait_in = [&]() -> bool {
        const bool ok = mbar_wait(&bar_in, ph_in, status);
        ph_in ^= 1;
        if (t == 0) in_pending = false;
        return ok;
    };
    // this thread's log_alpha pairs (channels c0, c0 + 1; the 8 tokens of its warp) of one 64-channel half,
    // loaded one half ahead of their use (zero past the item's n tokens)
    float2 nla[8];
    auto load_la_half = [&](int2 l, int hh, int hf) {
        const size_t row0 = static_cast<size_t>(l.x) * H + hh;
        const int c0 = 64 * hf + 2 * lane;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = 8 * w + j;
            nla[j] = r < l.y ? ld_once_f2(lag + (row0 + static_cast<size_t>(r) * H) * kDK + c0) : make_float2(0.f, 0.f);
        }
    };

    // everything above is private set-up; the chunk table and the inputs come from earlier launches
    grid_dependency_wait();
    // Item it = c H + h; a CTA's next item is gridDim.x further on, so (c, h) advance by
    // (gridDim.x / H, gridDim.x % H) with a carry, without a 64-bit division per item.  Item c takes the
    // window's chunk n_valid - 1 - c: the chunks are prepared last to first, so that the state pass, which
    // walks every chain from its first chunk, finds the packets written last (its first ones) still in L2.
    // The window's valid chunks (n > 0) are a prefix of its table, the rest lying past the batch's last
    // chunk, so a binary search over the table finds their count n_valid.
    // entry(c): the chunk table entry {first token, valid tokens} of item c (n = 0: none).
    const long long n_chunks_win = n_items / H;
    long long n_valid = 0;
    for (long long hi = n_chunks_win; n_valid < hi;) {
        const long long mid = (n_valid + hi) / 2;
        if (chunk_tab[mid].y > 0) n_valid = mid + 1; else hi = mid;
    }
    const int step_c = static_cast<int>(gridDim.x) / H, step_h = static_cast<int>(gridDim.x) % H;
    auto entry = [&](long long ch) -> int2 { return ch < n_valid ? chunk_tab[n_valid - 1 - ch] : make_int2(0, 0); };
    long long item = blockIdx.x;
    long long c = static_cast<int>(blockIdx.x) / H;
    int h = static_cast<int>(blockIdx.x) % H;
    int2 loc = entry(c);
    bool valid = loc.y > 0;
    if (valid) {
        if (t == 0) issue_kq(loc.x, h, 0);
        load_la_half(loc, h, 0);
    }

    while (valid) {
        const int n = loc.y;
        uint8_t* pkt = packets + static_cast<size_t>((n_valid - 1 - c) * H + h) * P::BYTES;
        const long long nitem = item + gridDim.x;   // this CTA's next item
        long long nc = c + step_c;
        int nh = h + step_h;
        if (nh >= H) {
            nh -= H;
            ++nc;
        }
        const int2 nloc = entry(nc);
        const bool nvalid = nloc.y > 0;
        // beta (threads 0..63) and the MXFP8 scale words (threads 64..255) of the chunk's rows go to shared
        // memory only later in the column pass, so that no thread waits for these loads before its first barrier
        float beta_r = 0.f;
        uint32_t scale_w = 0x7F7F7F7Fu;   // scale 1.0 past the item's end
        if (t < 64) {
            if (t < n) beta_r = beta[(static_cast<size_t>(loc.x) + t) * H + h];
            if (nvalid && t < nloc.y) prefetch_l2(beta + (static_cast<size_t>(nloc.x) + t) * H + nh);
        } else if constexpr (MX) {
            const int which = (t - 64) >> 6, rr = (t - 64) & 63;
            const size_t row = (static_cast<size_t>(loc.x) + rr) * H + h;
            if (rr < n) {
                if (which == 0) scale_w = ld_once_u32(q_scale + 4 * row);
                else if (which == 1) scale_w = ld_once_u32(k_scale + 4 * row);
                else scale_w = DV == 128 ? ld_once_u32(v_scale + 4 * row) : (0x7F7F0000u | ld_once_u16(v_scale + 2 * row));
            }
        }
        // the previous item's packet staging (OPB, QG, KG) must have been read out before this column pass
        // writes there: each warp's lane 0 waits for the bulk copies it issued, before the first barrier below

        // ---------------- column pass, one 64-channel half at a time: thread = (channel pair, the 8 tokens
        // of its warp); each half ends with its share of product A (K = 64 channels)
        bool fail = false;
        for (int hf = 0; hf < 2; ++hf) {
            const int c0 = 64 * hf + 2 * lane, tq = w >> 1;
            float2 p[8];
            uint32_t kb8[8], qb8[8], vb8[8];
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = 8 * w + j;
                kb8[j] = qb8[j] = vb8[j] = 0u;
                p[j] = nla[j];   // log_alpha, loaded one half ahead (k, q: the staged TMA tiles)
                if constexpr (MX) {   // MXFP8 v codes of this half with plain loads
                    const size_t rr = (static_cast<size_t>(loc.x) + r) * H + h;   // (token, head) row
                    if (r < n && c0 < DV) vb8[j] = ld_once_u16(vg + rr * DV + c0);
                }
            }
            if (hf == 0) load_la_half(loc, h, 1);   // lands while this half's operands are made
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (8 * w + j < n) acc = __fadd2_rn(acc, make_float2(floor_log_decay(p[j].x), floor_log_decay(p[j].y)));
                p[j] = acc;
            }
            *reinterpret_cast<float2*>(tot + w * 64 + 2 * lane) = acc;
            if constexpr (MX) {   // the shared scales of the chunk's tokens as fp32, needed from here on
                if (hf == 0 && t >= 64)
                    reinterpret_cast<float4*>(sm + ps::SCF)[t - 64] =
                        make_float4(e8m0_to_f32(scale_w & 0xFFu), e8m0_to_f32((scale_w >> 8) & 0xFFu),
                                    e8m0_to_f32((scale_w >> 16) & 0xFFu), e8m0_to_f32(scale_w >> 24));
            }
            if (hf == 0 && lane == 0) bulk_wait_read0();
            {   // this half's k and q tiles have landed (bf16), and product A's first half has finished reading
                // OPB (second half)
                bool ok = wait_in();
                if (hf == 1) {
                    ok = mbar_wait(&bar_mma, ph_mma, status) && ok;
                    ph_mma ^= 1;
                }
                if (__syncthreads_or(!ok)) { fail = true; break; }
            }
            if (w & 1) {   // second half of the tile: add the first half's total
                const float2 ob = *reinterpret_cast<const float2*>(tot + (w - 1) * 64 + 2 * lane);
#pragma unroll
                for (int j = 0; j < 8; ++j) { p[j].x += ob.x; p[j].y += ob.y; }
            }
            // p[j] = g_r - b_tq: the log-decay inside the tile up to r
            float bx[5], by[5];
            bx[0] = 0.f; by[0] = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 t0 = *reinterpret_cast<const float2*>(tot + (2 * i) * 64 + 2 * lane);
                const float2 t1 = *reinterpret_cast<const float2*>(tot + (2 * i + 1) * 64 + 2 * lane);
                bx[i + 1] = bx[i] + t0.x + t1.x;
                by[i + 1] = by[i] + t0.y + t1.y;
            }
            // anchors of this thread's tile, selected with compile-time indices (no local-memory arrays)
            float btx = 0.f, bty = 0.f, bnx = 0.f, bny = 0.f;   // b_t and b_{t+1}
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (i == tq) { btx = bx[i]; bty = by[i]; bnx = bx[i + 1]; bny = by[i + 1]; }
            const float ebx = exp_ftz(btx), eby = exp_ftz(bty);                 // e^{b_t}
            const float ftx = exp_ftz(bnx - btx), fty = exp_ftz(bny - bty);     // e^{b_{t+1}-b_t}
            const float ecx = exp_ftz(bx[4] - bnx), ecy = exp_ftz(by[4] - bny); // e^{g_C-b_{t+1}}
            float dvx[4], dvy[4];   // e^{b_i - b_{t+1}}, i > t
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                dvx[i] = i > tq ? exp_ftz(bx[i] - bnx) : 0.f;
                dvy[i] = i > tq ? exp_ftz(by[i] - bny) : 0.f;
            }
            if (w == 7)
                *reinterpret_cast<float2*>(pkt + P::G + c0 * 4) = make_float2(exp_ftz(bx[4]), exp_ftz(by[4]));

            // -K gamma and Kdec along the 8 tokens, packed to bf16 pairs of consecutive tokens as they are made
            uint32_t tkw[2][4], tdw[2][4];
            float2 tkp = make_float2(0.f, 0.f), tdp = make_float2(0.f, 0.f);
            const float2 ft2 = make_float2(ftx, fty), eb2 = make_float2(ebx, eby), ec2 = make_float2(ecx, ecy);
            const uint32_t kk = static_cast<uint32_t>((c0 & 63) >> 3), kb = static_cast<uint32_t>(c0 & 7) * 2;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = 8 * w + j;
                // rows past the sequence end (n <= r) hold zero inputs: their log-decay and beta are zero, so
                // they add nothing to A, W, U, Kdec^T U' or the state, and their own Q gamma / Aqk rows are never
                // stored as outputs
                float2 kf, qf;
                if constexpr (MX) {   // code x shared scale of the 32-channel block holding c0
                    const float* scf = reinterpret_cast<const float*>(sm + ps::SCF) + (c0 >> 5);
                    // rows past n hold other tokens' (finite) codes, which nothing below lets through
                    const uint32_t kc = *reinterpret_cast<const uint16_t*>(kq_stage + r * 64 + (c0 & 63));
                    const uint32_t qc = *reinterpret_cast<const uint16_t*>(kq_stage + kKQ + r * 64 + (c0 & 63));
                    kf = __fmul2_rn(e4m3x2_to_f2(kc), f2(scf[4 * (64 + r)]));
                    qf = __fmul2_rn(e4m3x2_to_f2(qc), f2(scf[4 * r]));
                    if (c0 < DV) {   // V as product B's MN-major operand
                        const float2 vf = __fmul2_rn(e4m3x2_to_f2(vb8[j]), f2(scf[4 * (128 + r)]));
                        st_b32(sm + ps::VOP + (c0 >> 6) * 8192 + (r >> 3) * 1024 + (r & 7) * 128 +
                                   ((kk ^ static_cast<uint32_t>(r & 7)) << 4) + kb,
                               pack2(vf));
                    }
                } else {   // rows past n hold other tokens' (finite) values, which nothing below lets through
                    kf = bf2_to_f2(*reinterpret_cast<const uint32_t*>(sm + ps::VOP + r * 128 + (c0 & 63) * 2));
                    qf = bf2_to_f2(*reinterpret_cast<const uint32_t*>(sm + ps::VOP + 8192 + r * 128 + (c0 & 63) * 2));
                }
                const float2 pl = __fmul2_rn(p[j], f2(kLog2e));
                const float2 E = make_float2(ex2_approx(pl.x), ex2_approx(pl.y));     // e^{g_r - b_t} <= 1
                const float2 I = make_float2(ex2_approx(-pl.x), ex2_approx(-pl.y));   // e^{b_t - g_r} <= e^80.09
                const float2 F = __fmul2_rn(ft2, I);                                  // e^{b_{t+1} - g_r} <= 1
                const float2 G = __fmul2_rn(eb2, E);                                  // e^{g_r}
                const uint32_t sw = ((kk ^ static_cast<uint32_t>(r & 7)) << 4) + kb;  // row r, rows 8 apart agree
                // row side of A / Aqk (this half's K atom)
                st_b32(sm + ps::OPB + r * 128 + sw, pack2(__fmul2_rn(kf, E)));
                st_b32(sm + ps::OPB + (64 + r) * 128 + sw, pack2(__fmul2_rn(qf, E)));
                // key side: own tile (diagonal) and the variants of later row tiles (variant i: rows 8 i (i+1) + r)
                st_b32(sm + ps::BVAR + (8 * tq * (tq + 1) + r) * 128 + sw, pack2(__fmul2_rn(kf, I)));
                const float2 kF = __fmul2_rn(kf, F);
#pragma unroll
                for (int i = 1; i < 4; ++i)
                    if (i > tq)
                        st_b32(sm + ps::BVAR + (8 * i * (i + 1) + r) * 128 + sw,
                               pack2(__fmul2_rn(kF, make_float2(dvx[i], dvy[i]))));
                // Q * gamma, rows 64..127 of the packet's [-W; Q gamma] (atom hf)
                st_b32(sm + ps::QG + hf * 8192 + r * 128 + sw, pack2(__fmul2_rn(qf, G)));
                const float2 tk2 = __fmul2_rn(make_float2(-kf.x, -kf.y), G);   // -K gamma
                const float2 td2 = __fmul2_rn(kF, ec2);                        // Kdec = K e^{g_C - g}
                if (j & 1) {
                    tkw[0][j >> 1] = pack_bf16x2(tkp.x, tk2.x); tkw[1][j >> 1] = pack_bf16x2(tkp.y, tk2.y);
                    tdw[0][j >> 1] = pack_bf16x2(tdp.x, td2.x); tdw[1][j >> 1] = pack_bf16x2(tdp.y, td2.y);
                } else {
                    tkp = tk2;
                    tdp = td2;
                }
            }
            // rows c of the transposed operands (8 tokens = one 16-byte chunk): lanes 4..7 of each quarter warp
            // take their odd channel first, so that the 8 lanes of a quarter warp hit 8 different bank groups.
            // -(K gamma)^T goes to KG; Kdec^T leaves for the packet straight from registers.
            {
                const bool odd_first = (lane >> 2) & 1;
                const uint4 k0 = make_uint4(tkw[0][0], tkw[0][1], tkw[0][2], tkw[0][3]);
                const uint4 k1 = make_uint4(tkw[1][0], tkw[1][1], tkw[1][2], tkw[1][3]);
                const uint4 d0 = make_uint4(tdw[0][0], tdw[0][1], tdw[0][2], tdw[0][3]);
                const uint4 d1 = make_uint4(tdw[1][0], tdw[1][1], tdw[1][2], tdw[1][3]);
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const int ch = it ^ static_cast<int>(odd_first);
                    const int c = c0 + ch;
                    const uint32_t sw = static_cast<uint32_t>((w ^ (c & 7)) << 4);   // 8-token chunk w of row c
                    *reinterpret_cast<uint4*>(sm + ps::KG + c * 128 + sw) = (ch ? k1 : k0);
                    st_global_v4(pkt + P::KD + c * 128 + sw, ch ? d1 : d0);
                }
            }
            if (hf == 0 && t < 64) bet[t] = beta_r;   // first read by the A epilogue
            fence_proxy_async_smem();
            __syncthreads();
            // ---------------- product A, this half: D[m, n] += RALL[m, :] . BVAR[n, :]  (M = 128, N = 160,
            // K = 64); the columns of variant i (row tile i's key side) are [8 i (i+1), 8 (i+1)(i+2))
            if (t == 0) {
                // VOP has been read: the second half's k and q tiles, then V (product B's operand); MXFP8: the
                // second half's code tiles have been read, so the next item's first ones follow.  The loads go
                // first: issuing the products holds this thread for several hundred cycles.
                if (hf == 0) issue_kq(loc.x, h, 1);
                else if (!MX) issue_v(loc.x, h);
                else if (nvalid) issue_kq(nloc.x, nh, 0);
                tc_fence_after();
                const uint32_t ra = smem_u32(sm + ps::OPB), bv = smem_u32(sm + ps::BVAR);
                const uint32_t idesc = idesc_bf16(128, 160);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_f16(tm, sdesc_k_sw128(ra + ks * 32), sdesc_k_sw128(bv + ks * 32), idesc, hf > 0 || ks > 0);
                umma_commit(&bar_mma);
            }
        }
        if (fail) break;
        {
            const bool ok = mbar_wait(&bar_mma, ph_mma, status);
            if (__syncthreads_or(!ok)) break;
        }
        ph_mma ^= 1;
        tc_fence_after();

        // ---------------- TMEM -> fp32 A (strict lower, beta rows) and bf16 Aqk (inclusive lower, the packet's layout).
        // Lane quarter qw holds the rows of tiles t0 = 2 (qw & 1) and t0 + 1 (K rows for qw < 2, Q rows
        // otherwise).  Their variant columns form 2 t0 + 3 chunks of 16 (t0 + 1 of tile t0, t0 + 2 of tile
        // t0 + 1), spread over the lane quarter's two warps, at most four per warp, in two rounds of two.
        {
            const int qw = w & 3, sub = w >> 2;
            const int t0 = 2 * (qw & 1), nchunk = 2 * t0 + 3;
            const int r = (32 * qw + lane) & 63;
            const bool is_q = qw >= 2;
            const float br = bet[r];
#pragma unroll
            for (int rd = 0; rd < 2; ++rd) {   // two rounds of two 16-column chunks: loads in flight, one wait
                float v4[32];
                int tile_of[2], cb_of[2];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int j = sub + 2 * (2 * rd + hh);
                    tile_of[hh] = j < t0 + 1 ? t0 : t0 + 1;
                    cb_of[hh] = 16 * (j < t0 + 1 ? j : j - t0 - 1);
                    if (j < nchunk) {
                        tmem_ld16(tm + (static_cast<uint32_t>(32 * qw) << 16) + 8 * tile_of[hh] * (tile_of[hh] + 1) +
                                      cb_of[hh],
                                  *reinterpret_cast<float(*)[16]>(v4 + 16 * hh));
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) v4[16 * hh + e] = 0.f;
                    }
                }
                tmem_wait_ld_regs<32>(v4);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int cb = cb_of[hh];
                    const float* v = v4 + 16 * hh;
                    if (sub + 2 * (2 * rd + hh) < nchunk && (r >> 4) == tile_of[hh]) {   // the lane's row is in the tile
                        if (is_q) {
                            float o8[8];
#pragma unroll
                            for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                                for (int j = 0; j < 8; ++j) o8[j] = (cb + 8 * hf + j <= r) ? v[8 * hf + j] : 0.f;
                                const int sc = (cb >> 3) + hf;
                                *reinterpret_cast<uint4*>(sm + ps::IAQ + (64 + r) * 128 + ((sc ^ (r & 7)) << 4)) =
                                    pack8(o8);
                            }
                        } else if ((cb >> 4) == (r >> 4)) {   // diagonal block: transposed, strict lower part only
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const int s2 = cb + j;
                                if (s2 < r) AM[s2 * LDM + r] = br * v[j];
                            }
                        } else {                              // off-diagonal block: row-major
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4)
                                reinterpret_cast<float4*>(AM + r * LDM + cb)[q4] = make_float4(
                                    br * v[4 * q4], br * v[4 * q4 + 1], br * v[4 * q4 + 2], br * v[4 * q4 + 3]);
                        }
                    }
                }
            }
        }
        tc_fence_before();
        // ---------------- X = (I + A)^-1 by blocked forward substitution over 16 x 16 tiles, each lane quarter's
        // warps on their own: the K-row warps of quarter kq (warps kq and kq + 4, rows 32 kq .. 32 kq + 31 of A)
        // invert the quarter's two diagonal blocks and merge them (levels 0 and 1) as soon as their own rows of
        // A are written, while the Q-row warps (quarters 2, 3) finish Aqk, send it, and clear X above its
        // diagonal blocks.  Level 2 follows a CTA barrier.
        const int fg = lane >> 2, ft = lane & 3;   // fragment row group and column pair of this lane
        if ((w & 3) >= 2) {
            fence_proxy_async_smem();   // Aqk leaves by a bulk copy
            named_bar_sync(1, 128);     // the four Q-row warps have written Aqk
            // Aqk and Q gamma are final: warp 2 sends them to the packet (waited for before the next column pass)
            if (t == 64) {
                bulk_s2g(pkt + P::AQ, sm + ps::IAQ + 8192, 8192);
                bulk_s2g(pkt + P::AW + 8192, sm + ps::QG, 8192);
                bulk_s2g(pkt + P::AW + 16384 + 8192, sm + ps::QG + 8192, 8192);
                bulk_commit();
            }
            const int zt = 32 * (2 * (w >> 2) + (w & 1)) + lane;   // 0..127 over warps 2, 3, 6, 7
            for (int e = zt; e < 64 * 64; e += 128) {   // the blocks above the diagonal are zero
                const int r = e >> 6, c = e & 63;
                if ((c >> 4) > (r >> 4)) XF[r * LDX + c] = 0.f;
            }
        } else {
            const int kq = w & 3, hb = w >> 2;   // lane quarter (0, 1) and which of its two warps
            if (kq == 1) named_bar_arrive(4, 128);   // rows 32..63 of A (A_10 of level 2) are written
            named_bar_sync(2 + kq, 64);          // this quarter's rows of A are written
            {   // level 0: diagonal block 2 kq + hb by forward substitution, lane = column, the column held in
                // registers; a column of A comes as float4 broadcasts of a row of the transposed block
                const int o0 = 16 * (2 * kq + hb), col = lane & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) x[r] = (r == col) ? 1.f : 0.f;
                float4 cur[4], nxt[4];
#pragma unroll
                for (int r4 = 0; r4 < 4; ++r4) cur[r4] = reinterpret_cast<const float4*>(AM + o0 * LDM + o0)[r4];
#pragma unroll
                for (int m = 0; m < 15; ++m) {
                    if (m + 1 < 15) {
#pragma unroll
                        for (int r4 = (m + 2) >> 2; r4 < 4; ++r4)
                            nxt[r4] = reinterpret_cast<const float4*>(AM + (o0 + m + 1) * LDM + o0)[r4];
                    }
                    const float xm = x[m];
#pragma unroll
                    for (int r4 = (m + 1) >> 2; r4 < 4; ++r4) {
                        const float4 a = cur[r4];
                        if (4 * r4 + 0 > m) x[4 * r4 + 0] = fmaf(-a.x, xm, x[4 * r4 + 0]);
                        if (4 * r4 + 1 > m) x[4 * r4 + 1] = fmaf(-a.y, xm, x[4 * r4 + 1]);
                        if (4 * r4 + 2 > m) x[4 * r4 + 2] = fmaf(-a.z, xm, x[4 * r4 + 2]);
                        if (4 * r4 + 3 > m) x[4 * r4 + 3] = fmaf(-a.w, xm, x[4 * r4 + 3]);
                    }
#pragma unroll
                    for (int r4 = 0; r4 < 4; ++r4) cur[r4] = nxt[r4];
                }
                if (lane < 16) {
#pragma unroll
                    for (int r = 0; r < 16; ++r) XF[(o0 + r) * LDX + o0 + col] = x[r];
                }
            }
            named_bar_sync(2 + kq, 64);   // both diagonal blocks of the quarter are inverted
            // Levels 1 and 2 merge two inverted diagonal blocks: X_10 = -X_11 (A_10 X_00).  The products are
            // 16- and 32-row tiles, below the tensor-core MMA's smallest M, so they run as warp-level tf32
            // m16n8k8 MMAs with fp32 accumulation on fragments loaded straight from shared memory.
            {   // level 1: 16 -> 32, pair kq (rows 32 kq + 16 .., cols 32 kq ..), column tile hb of 8
                const int nt = hb, rb = 32 * kq + 16, c0 = 32 * kq;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    if (ks < nt) continue;   // X_00 is zero above its diagonal
                    const uint32_t a[4] = {to_tf32(AM[(rb + fg) * LDM + c0 + 8 * ks + ft]),
                                           to_tf32(AM[(rb + fg + 8) * LDM + c0 + 8 * ks + ft]),
                                           to_tf32(AM[(rb + fg) * LDM + c0 + 8 * ks + ft + 4]),
                                           to_tf32(AM[(rb + fg + 8) * LDM + c0 + 8 * ks + ft + 4])};
                    const uint32_t b[2] = {to_tf32(XF[(c0 + 8 * ks + ft) * LDX + c0 + 8 * nt + fg]),
                                           to_tf32(XF[(c0 + 8 * ks + ft + 4) * LDX + c0 + 8 * nt + fg])};
                    mma_tf32(d, a, b);
                }
                float* tt = TT + 16 * kq * LDTT + 8 * nt;
                *reinterpret_cast<float2*>(tt + fg * LDTT + 2 * ft) = make_float2(d[0], d[1]);
                *reinterpret_cast<float2*>(tt + (fg + 8) * LDTT + 2 * ft) = make_float2(d[2], d[3]);
                __syncwarp();
                float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    const uint32_t a[4] = {to_tf32(XF[(rb + fg) * LDX + rb + 8 * ks + ft]),
                                           to_tf32(XF[(rb + fg + 8) * LDX + rb + 8 * ks + ft]),
                                           to_tf32(XF[(rb + fg) * LDX + rb + 8 * ks + ft + 4]),
                                           to_tf32(XF[(rb + fg + 8) * LDX + rb + 8 * ks + ft + 4])};
                    const uint32_t b[2] = {to_tf32(tt[(8 * ks + ft) * LDTT + fg]), to_tf32(tt[(8 * ks + ft + 4) * LDTT + fg])};
                    mma_tf32(e, a, b);
                }
                float* xo = XF + rb * LDX + c0 + 8 * nt + 2 * ft;
                xo[fg * LDX] = -e[0];
                xo[fg * LDX + 1] = -e[1];
                xo[(fg + 8) * LDX] = -e[2];
                xo[(fg + 8) * LDX + 1] = -e[3];
            }
            if (kq == 0) {
                // Level 2's first product, T = A_10 X_00 (32 x 32, K = 32), needs only X_00 and rows 32..63 of A,
                // so quarter 0's warps form it (row tile hb) while quarter 1 is still inverting X_11.  T goes
                // to rows 0..31 of A, which levels 0 and 1 of quarter 0 no longer read.
                named_bar_sync(4, 128);   // both warps of quarter 0 are through level 1; quarter 1 has arrived
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        if (ks < nt) continue;   // X_00 is zero above its diagonal
                        const int ra = 32 + 16 * hb + fg;
                        const uint32_t a[4] = {to_tf32(AM[ra * LDM + 8 * ks + ft]), to_tf32(AM[(ra + 8) * LDM + 8 * ks + ft]),
                                               to_tf32(AM[ra * LDM + 8 * ks + ft + 4]),
                                               to_tf32(AM[(ra + 8) * LDM + 8 * ks + ft + 4])};
                        const uint32_t b[2] = {to_tf32(XF[(8 * ks + ft) * LDX + 8 * nt + fg]),
                                               to_tf32(XF[(8 * ks + ft + 4) * LDX + 8 * nt + fg])};
                        mma_tf32(d, a, b);
                    }
                    float* ts = TS + 16 * hb * LDTT + 8 * nt;
                    *reinterpret_cast<float2*>(ts + fg * LDTT + 2 * ft) = make_float2(d[0], d[1]);
                    *reinterpret_cast<float2*>(ts + (fg + 8) * LDTT + 2 * ft) = make_float2(d[2], d[3]);
                }
            }
        }
        __syncthreads();
        {   // level 2: 32 -> 64, X_10 = -X_11 T: row tile mt of 16 and column tile nt of 8
            const int nt = w & 3, mt = w >> 2;
            float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                if (ks >= 2 * (mt + 1)) continue;   // X_11 is zero above its diagonal
                const int ra = 32 + 16 * mt + fg;
                const uint32_t a[4] = {to_tf32(XF[ra * LDX + 32 + 8 * ks + ft]),
                                       to_tf32(XF[(ra + 8) * LDX + 32 + 8 * ks + ft]),
                                       to_tf32(XF[ra * LDX + 32 + 8 * ks + ft + 4]),
                                       to_tf32(XF[(ra + 8) * LDX + 32 + 8 * ks + ft + 4])};
                const uint32_t b[2] = {to_tf32(TS[(8 * ks + ft) * LDTT + 8 * nt + fg]),
                                       to_tf32(TS[(8 * ks + ft + 4) * LDTT + 8 * nt + fg])};
                mma_tf32(e, a, b);
            }
            float* xo = XF + (32 + 16 * mt) * LDX + 8 * nt + 2 * ft;
            xo[fg * LDX] = -e[0];
            xo[fg * LDX + 1] = -e[1];
            xo[(fg + 8) * LDX] = -e[2];
            xo[(fg + 8) * LDX + 1] = -e[3];
        }
        __syncthreads();
        // [X; X] diag(beta) as product B's A operand (K = 64 tokens, K-major): rows 64..127 repeat rows 0..63, so
        // that the lanes of all four TMEM quarters hold -W and U rows for the epilogue
#pragma unroll
        for (int e = t; e < 64 * 8; e += NT) {
            const int m = e >> 3, uc = e & 7;
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = XF[m * LDX + 8 * uc + j] * bet[8 * uc + j];
            const uint4 pk8 = pack8(v);
            const uint32_t off = static_cast<uint32_t>(m * 128 + ((uc ^ (m & 7)) << 4));
            *reinterpret_cast<uint4*>(sm + ps::OPB + off) = pk8;
            *reinterpret_cast<uint4*>(sm + ps::OPB + 8192 + off) = pk8;
        }
        fence_proxy_async_smem();
        {   // V of this item has landed (bf16 inputs: its TMA tile)
            const bool ok = MX || wait_in();
            if (__syncthreads_or(!ok)) break;
        }
        tc_fence_after();

        // ---------------- phase B: D[m, n] = [X; X] diag(beta) [m, :] . B[n, :]  (K = 64 tokens): the K part
        // (N = 128, B = -(K gamma)^T) gives -W, the V part (N = DV, B = V MN-major) gives U
        if (t == 0) {
            const uint32_t xa = smem_u32(sm + ps::OPB), kb = smem_u32(sm + ps::KG), vb = smem_u32(sm + ps::VOP);
            const uint32_t idk = idesc_bf16(128, 128), idv = idesc_bf16(128, DV, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_f16(tm, sdesc_k_sw128(xa + ks * 32), sdesc_k_sw128(kb + ks * 32), idk, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_f16(tm + 128, sdesc_k_sw128(xa + ks * 32), sdesc_mn_sw128(vb + ks * 2048, 8192), idv, ks > 0);
            umma_commit(&bar_mma);
        }
        {
            const bool ok = mbar_wait(&bar_mma, ph_mma, status);
            if (__syncthreads_or(!ok)) break;
        }
        ph_mma ^= 1;
        tc_fence_after();
        // product B has read VOP
        if (nvalid) {   // bf16: VOP is free again for the next item's first k, q tiles; and its first log_alpha half
            if (!MX && t == 0) issue_kq(nloc.x, nh, 0);
            load_la_half(nloc, nh, 0);
        }

        // ---------------- epilogue: -W (lane quarters 0, 1) and U (lane quarters 2, 3, the repeated rows), straight
        // from TMEM into the packet staging (-W over OPB, U at OPB + 16384).  Each warp stages the 32 rows of its
        // lane quarter in one 64-column atom (4 KB) and sends them with its own bulk copy at once, so no CTA
        // barrier precedes the packet store.
        {
            const int qw = w & 3, cg = w >> 2;   // qw 0, 1: -W atom cg; qw 2, 3: U atom cg
            const bool upart = qw >= 2;
            const int m = (32 * qw + lane) & 63;   // token row
            if (!upart || cg < DV / 64) {
                const uint32_t col = upart ? 128 + 64 * cg : 64 * cg;
                const uint32_t lane_base = tm + (static_cast<uint32_t>(32 * qw) << 16) + col;
                uint8_t* const stg = sm + ps::OPB + (upart ? 16384 : 0) + cg * 8192;
#pragma unroll
                for (int hq = 0; hq < 2; ++hq) {
                    float vv[32];
                    tmem_ld16(lane_base + 32 * hq, *reinterpret_cast<float(*)[16]>(vv));
                    tmem_ld16(lane_base + 32 * hq + 16, *reinterpret_cast<float(*)[16]>(vv + 16));
                    tmem_wait_ld_regs<32>(vv);
#pragma unroll
                    for (int sub = 0; sub < 4; ++sub) {
                        float o8[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) o8[j] = vv[8 * sub + j];
                        *reinterpret_cast<uint4*>(stg + m * 128 + (((4 * hq + sub) ^ (m & 7)) << 4)) = pack8(o8);
                    }
                }
                tc_fence_before();   // this warp's TMEM loads precede the next item's products (barriers in between)
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int r0 = 32 * (qw & 1);   // first token row of this warp
                    uint8_t* gdst = pkt + (upart ? P::U + cg * 8192 : P::AW + cg * 16384) + r0 * 128;
                    bulk_s2g(gdst, stg + r0 * 128, 4096);
                    bulk_commit();   // waited for (read out) before the next column pass's first barrier
                }
            }
        }
        item = nitem;
        c = nc;
        loc = nloc;
        h = nh;
        valid = nvalid;
    }
    if (t == 0 && in_pending) mbar_wait(&bar_in, ph_in, nullptr);   // never leave a TMA write in flight
    if (lane == 0) bulk_wait0();                                    // nor a packet store
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tm, 256);
}

// ------------------------------------------------------------------------------------------------
// inter-chunk state pass
template <int DV, int DVS>
struct SCfg {
    static constexpr int NEW = DVS >= 64 ? 16 : 8;        // epilogue warps (NEW/4 share each TMEM lane quarter)
    static constexpr int NCW = DVS * 4 / NEW;              // state columns per epilogue warp (>= 16)
    static constexpr int NT = 32 * (NEW + 2);              // + producer warp + MMA warp
    // Full 128-column slices run all three products transposed, with the state columns on the M side:
    // D1^T = S^T [-W; Q gamma]^T (A = S^T in TMEM), D2^T = U'^T Kdec and O^T += U'^T Aqk^T, so that D1^T's
    // TMEM lanes are state columns; warps 0..7 then form U' and warps 8..15 read O, 32 tokens per warp in
    // the fragment layout of 16-lane TMEM loads and 8 x 8 matrix loads and stores.  Narrower slices cannot
    // fill M = 128 and keep D1 = [-W; Q gamma] S and D2 = Kdec^T U' (S and U' as MN-major B operands).
    static constexpr bool TR = DVS == 128;
    // Narrower slices stage S and U' MN-major (row = channel / token) in blocks of 64 columns; a 32-column
    // slice fills half of one block (a product with N = 32 reads just those columns).  The transposed path
    // stages U'^T K-major (row = state column) and keeps S out of shared memory (SOP unused)
    static constexpr int DVA = DVS >= 64 ? DVS : 64;
    static constexpr bool TMA_O = DVS >= 64;               // whole 64-column O tiles leave by tensor stores
    static constexpr int NST = DVS == 32 ? 3 : 2;
    static constexpr uint32_t U_BYTES = DVS >= 64 ? DVS * 128 : 8192;   // whole 64-column atoms of U
    // stage: the packet's parts for this slice (Aqk right after Kdec^T, as in the packet)
    static constexpr uint32_t AW = 0, KD = 32768, AQ = 49152, U = 57344, G = U + U_BYTES;
    static constexpr uint32_t STAGE = ((G + 512 + 1023) / 1024) * 1024;
    static constexpr uint32_t SOP = NST * STAGE;      // S as B operand (N = DVS, K = 128)
    static constexpr uint32_t UOP = SOP + DVA * 256;  // U' as B operand (N = DVS, K = 64); transposed: U'^T as A
    // O tile staging for the tensor store, [DVS/64][64 tokens][128 B] with the 128B swizzle (slices of whole
    // 64-column atoms only; narrower slices store O from registers)
    static constexpr uint32_t OST = UOP + DVA * 128;
    static constexpr uint32_t BYTES = OST + (TMA_O ? DVS * 128 : 0);
    // TMEM: D1 double-buffered at columns [0, DVS) and [2 DVS, 3 DVS), D2 at [DVS, 2 DVS); transposed path:
    // S^T in bf16 at [3 DVS, 3 DVS + 64)
    static constexpr uint32_t S_LBO = 128 * 128;      // MN-major: 64 columns x 128 K rows per block
    static constexpr uint32_t U_LBO = 64 * 128;       // MN-major: 64 columns x 64 K rows per block
    static constexpr uint32_t TMEM_COLS = 3 * DVS <= 128 ? 128 : (3 * DVS <= 256 ? 256 : 512);
    // Transposed path: S^T in bf16 (lane = state column, two channels per 32-bit column) as product 1's A
    // operand in TMEM, so that S never passes through shared memory
    static constexpr uint32_t SA_COL = 3 * DVS;
    static __host__ __device__ constexpr uint32_t d1col(int ci) { return (ci & 1) ? 2 * DVS : 0; }
    static_assert(BYTES + 1024 <= 232448, "one CTA per SM");
    static_assert(!TR || SA_COL + kDK / 2 <= TMEM_COLS, "S^T operand inside the TMEM allocation");
    static_assert(STAGE % 1024 == 0 && SOP % 1024 == 0 && UOP % 1024 == 0 && OST % 1024 == 0 && S_LBO % 1024 == 0,
                  "128B-swizzle operands and tiles on 1024-byte atoms");
};

template <int DV, int DVS>
__global__ void __launch_bounds__(SCfg<DV, DVS>::NT, 1)
state_bf16_kernel(const uint8_t* __restrict__ packets, const int32_t* __restrict__ cu_seqlens,
                  const int32_t* __restrict__ cu_chunks, int n_seqs, int H, long long win_lo, long long win_hi,
                  const float* __restrict__ initial_state, __nv_bfloat16* __restrict__ o,
                  const __grid_constant__ CUtensorMap map_o,
                  float* __restrict__ final_state, float* __restrict__ final_transition, int ckpt_stride,
                  float* __restrict__ checkpoints, const int32_t* __restrict__ ckpt_cu, float* __restrict__ carry,
                  int* status) {
    using C = SCfg<DV, DVS>;
    using P = Pk<DV>;
    constexpr int NST = C::NST, NCW = C::NCW, NEW = C::NEW, NSV = DV / DVS, CW = DV + kDK;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    __shared__ __align__(8) uint64_t full[NST], empty[NST], d1_full, d2_full, o_full, s_ready, up_ready;
    __shared__ uint32_t tmem_slot;
    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    grid_dependency_wait();   // the packets and the chunk index come from the launches before this one
    const int seq = blockIdx.x / H, h = blockIdx.x % H, slice = blockIdx.y;
    const bool trans = slice >= NSV;
    const int j0 = (trans ? slice - NSV : slice) * DVS;
    if (trans && !final_transition) return;
    const long long ch_lo = cu_chunks[seq], ch_hi = cu_chunks[seq + 1];
    const long long lo = ch_lo > win_lo ? ch_lo : win_lo;
    const long long hi = ch_hi < win_hi ? ch_hi : win_hi;
    const bool empty_seq = ch_lo == ch_hi;
    if (!(lo < hi) && !(empty_seq && win_lo == 0)) return;
    const bool first = empty_seq || ch_lo >= win_lo;
    const bool last = empty_seq || ch_hi <= win_hi;
    const int nch = static_cast<int>(hi > lo ? hi - lo : 0);
    const size_t sh = static_cast<size_t>(seq) * H + h;
    const long long seq_tok0 = cu_seqlens[seq];
    const long long seq_len = static_cast<long long>(cu_seqlens[seq + 1]) - seq_tok0;

    if (t == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + NEW);
        }
        mbar_init(&d1_full, 1);
        mbar_init(&d2_full, 1);
        mbar_init(&o_full, 1);
        mbar_init(&s_ready, NEW);
        mbar_init(&up_ready, NEW / 2);   // the warps that produce U'
        fence_barrier_init();
    }
    if (w == 0) {
        tmem_alloc(&tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_slot;

    if (w == NEW) {
        // ---------------- producer: packets -> shared-memory ring (bulk TMA)
        if (lane == 0) {
            int issued = 0;
            for (int ci = 0; ci < nch; ++ci) {
                const int st = ci % NST;
                if (!mbar_wait(&empty[st], ((ci / NST) & 1) ^ 1, status)) break;
                const uint8_t* pk = packets + static_cast<size_t>((lo + ci - win_lo) * H + h) * P::BYTES;
                uint8_t* sb = sm + st * C::STAGE;
                const uint32_t bytes = 32768 + 16384 + 512 + (trans ? 0u : 8192u + C::U_BYTES);
                mbar_arrive_expect_tx(&full[st], bytes);
                bulk_g2s(sb + C::AW, pk + P::AW, 32768, &full[st]);
                bulk_g2s(sb + C::KD, pk + P::KD, 16384, &full[st]);
                if (!trans) {
                    bulk_g2s(sb + C::AQ, pk + P::AQ, 8192, &full[st]);
                    bulk_g2s(sb + C::U, pk + P::U + (j0 / 64) * 8192, C::U_BYTES, &full[st]);
                }
                bulk_g2s(sb + C::G, pk + P::G, 512, &full[st]);
                issued = ci + 1;
            }
            // never leave a copy in flight: wait (bounded, quietly) for the last fill of every stage
            for (int ci = issued - NST < 0 ? 0 : issued - NST; ci < issued; ++ci)
                mbar_wait(&full[ci % NST], (ci / NST) & 1, nullptr);
        }
    } else if (w == NEW + 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, DVS, false, true);
            const uint32_t sop = smem_u32(sm + C::SOP), uop = smem_u32(sm + C::UOP);
            auto ubdesc = [&](int ks) -> uint64_t {   // U' as the B operand (K = 64 tokens)
                return sdesc_mn_sw128(uop + ks * 2048, C::U_LBO);
            };
            for (int ci = 0; ci < nch; ++ci) {
                const int st = ci % NST;
                if (!mbar_wait(&s_ready, ci & 1, status)) break;
                if (!mbar_wait(&full[st], (ci / NST) & 1, status)) break;
                tc_fence_after();
                const uint32_t sb = smem_u32(sm + st * C::STAGE);
                if constexpr (C::TR) {
                    // D1^T = S^T [-W; Q gamma]^T   (M = 128 state columns, N = 128 tokens: -W rows, then Q gamma
                    // rows; K = 128 channels), A = S^T in TMEM, B = the packet's K-major [-W; Q gamma]
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        umma_f16_ts(tm + C::d1col(ci), tm + C::SA_COL + ks * 8,
                                    sdesc_k_sw128(sb + C::AW + (ks >> 2) * 16384 + (ks & 3) * 32), idesc_bf16(128, 128),
                                    ks > 0);
                    umma_commit(&d1_full);
                    if (!mbar_wait(&up_ready, ci & 1, status)) break;
                    tc_fence_after();
                    // D2^T = U'^T Kdec   (M = 128 state columns, N = 128 channels, K = 64 tokens): A = U'^T K-major,
                    // B = the packet's Kdec^T rows (K-major)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_f16(tm + DVS, sdesc_k_sw128(uop + ks * 32), sdesc_k_sw128(sb + C::KD + ks * 32),
                                 idesc_bf16(128, 128), ks > 0);
                    umma_commit(&d2_full);
                    if (!trans) {
                        // O^T = (Q gamma S)^T + U'^T Aqk^T: D1^T columns 64..127 (M = 128, N = 64, K = 64 tokens)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            umma_f16(tm + C::d1col(ci) + 64, sdesc_k_sw128(uop + ks * 32),
                                     sdesc_k_sw128(sb + C::AQ + ks * 32), idesc_bf16(128, 64), true);
                        umma_commit(&o_full);
                    }
                } else {
                    // D1 = [-W; Q gamma] S   (M = 128, N = DVS, K = 128).  D1[ci] was last read as chunk ci - 2's O,
                    // before the O warps' s_ready arrival for chunk ci - 1.
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t ka = ks >> 2, kb = (ks & 3) * 32;
                        const uint64_t bdesc = sdesc_mn_sw128(sop + ks * 2048, C::S_LBO);
                        umma_f16(tm + C::d1col(ci), sdesc_k_sw128(sb + C::AW + ka * 16384 + kb), bdesc, idesc, ks > 0);
                    }
                    umma_commit(&d1_full);
                    if (!mbar_wait(&up_ready, ci & 1, status)) break;
                    tc_fence_after();
                    // D2 = Kdec^T U'   (M = 128, N = DVS, K = 64)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_f16(tm + DVS, sdesc_k_sw128(sb + C::KD + ks * 32), ubdesc(ks), idesc, ks > 0);
                    umma_commit(&d2_full);
                    if (!trans) {
                        // D1 rows 64..127 += Aqk U' (O = Q gamma S + Aqk U'): the A operand starts 64 rows into Kdec^T,
                        // so its rows 64..127 are Aqk; what it adds to rows 0..63 (U', already read) is never used
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            umma_f16(tm + C::d1col(ci), sdesc_k_sw128(sb + C::KD + 8192 + ks * 32), ubdesc(ks), idesc, true);
                        umma_commit(&o_full);
                    }
                }
                umma_commit(&empty[st]);
            }
        }
    } else {
        // ---------------- epilogue warps: lane quarter qw, columns [jw, jw + NCW) of the slice
        const int qw = w & 3, jw = (w >> 2) * NCW;
        // TMEM lane: channel of D2 and S; row of D1 (token row), or with transposed products the slice column
        // of D1^T, whose tokens [tk0, tk0 + 32) this warp takes (U' for warps 0..7, O for warps 8..15)
        const int i = 32 * qw + lane;
        const int tk0 = 32 * ((w >> 2) & 1);
        const uint32_t lane_base = tm + (static_cast<uint32_t>(32 * qw) << 16);
        // S[e]: element (channel i, slice column jw + e); transposed path: S^T, element (slice column i,
        // channel jw + e), the layout of D2^T and of product 1's A operand in TMEM.  srow / scol: the state
        // row (channel) and slice column of element e.
        float S[NCW];
        auto srow = [&](int e) { return C::TR ? jw + e : i; };
        auto scol = [&](int e) { return C::TR ? i : jw + e; };
        {
            const float* src = nullptr;
            size_t pitch = 0;
            if (!first) {
                src = carry + sh * kDK * CW + (trans ? DV : 0) + j0;
                pitch = CW;
            } else if (!trans && initial_state) {
                src = initial_state + sh * kDK * DV + j0;
                pitch = DV;
            }
            if constexpr (C::TR) {
#pragma unroll
                for (int e = 0; e < NCW; ++e) S[e] = src ? src[srow(e) * pitch + scol(e)] : 0.f;
            } else {
#pragma unroll
                for (int e = 0; e < NCW / 4; ++e) {
                    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (src) x = reinterpret_cast<const float4*>(src + i * pitch + jw)[e];
                    S[4 * e] = x.x; S[4 * e + 1] = x.y; S[4 * e + 2] = x.z; S[4 * e + 3] = x.w;
                }
            }
            if (first && trans) {
#pragma unroll
                for (int e = 0; e < NCW; ++e) S[e] = (srow(e) == j0 + scol(e)) ? 1.f : 0.f;
            }
        }
        // S as product 1's operand: MN-major rows of the B operand in shared memory, written 8 columns at a
        // time; transposed path: S^T in bf16 into TMEM (this warp's lanes, channels jw .. jw + NCW)
        auto write_sop = [&]() {
            if constexpr (C::TR) {
                float p16[NCW / 2];
#pragma unroll
                for (int e = 0; e < NCW / 2; ++e) p16[e] = __uint_as_float(pack_bf16x2(S[2 * e], S[2 * e + 1]));
                static_assert(NCW == 32, "one 16-column TMEM store per warp");
                tmem_st16(lane_base + C::SA_COL + jw / 2, p16);
                tmem_wait_st();
            } else {
#pragma unroll
                for (int j = 0; j < NCW; j += 8) {
                    float f8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f8[e] = S[j + e];
                    *reinterpret_cast<uint4*>(sm + C::SOP + sw128_mn_offset(jw + j, i, C::S_LBO)) = pack8(f8);
                }
            }
        };
        write_sop();
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_ready);
        const int ucol = (DVS >= 64 ? 0 : (j0 & 63)) + jw;   // this warp's first column inside the stage's U atoms
        // full chunks of whole-atom slices leave through a TMA tensor store of the O tile staged in OST
        const bool o_issuer = (w == (C::TR ? NEW / 2 : 2)) && lane == 0;
        // checkpoints: one after every cpe-th chunk of the sequence (ckpt_stride is a multiple of 64), counted
        // down without divisions in the loop; ck_slot is the next one's slot
        const int cpe = (!trans && ckpt_stride > 0 && checkpoints) ? ckpt_stride / 64 : 0;
        const int c_first = static_cast<int>(lo - ch_lo);
        int ck_wait = cpe > 0 ? cpe - c_first % cpe : 0;
        long long ck_slot = cpe > 0 ? static_cast<long long>(ckpt_cu[seq]) + c_first / cpe : 0;
        const long long ck_end = cpe > 0 ? static_cast<long long>(ckpt_cu[seq + 1]) : 0;
        for (int ci = 0; ci < nch; ++ci) {
            const int st = ci % NST;
            const uint8_t* sb = sm + st * C::STAGE;
            const int c = static_cast<int>(lo + ci - ch_lo);
            const long long rem = seq_len - static_cast<long long>(c) * 64;
            const int n = rem < 64 ? static_cast<int>(rem) : 64;
            const bool full_tma = C::TMA_O && !trans && n == 64;
            if (!mbar_wait(&full[st], (ci / NST) & 1, status)) break;
            if constexpr (C::TR) {
                if (w < NEW / 2) {
                    // U'^T = U^T - (W S)^T for state columns [32 qw, 32 qw + 32) and tokens [tk0, tk0 + 32), in the
                    // fragment layout: token block tb, lane half hh and token half bb make 16 x 8 tiles, each two
                    // 8 x 8 matrices (column half vh); U comes from the stage by transposing matrix loads, D1^T from
                    // TMEM by 16-lane loads, and U'^T goes to row v of the K-major operand by matrix stores.
                    const int mj = lane >> 3, mr = lane & 7;   // matrix j = 2 bb + vh, row mr: this lane's address
                    uint32_t uf[2][2][4];
#pragma unroll
                    for (int tb = 0; tb < 2; ++tb)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            if (!trans) {
                                const int v0 = 32 * qw + 16 * hh + 8 * (mj & 1), tok = tk0 + 16 * tb + 8 * (mj >> 1) + mr;
                                ldsm_x4_trans(smem_u32(sb + C::U + (v0 >> 6) * 8192 + tok * 128 +
                                                       ((((v0 & 63) >> 3) ^ (tok & 7)) << 4)),
                                              uf[tb][hh]);
                            } else {
                                uf[tb][hh][0] = uf[tb][hh][1] = uf[tb][hh][2] = uf[tb][hh][3] = 0u;
                            }
                        }
                    if (!mbar_wait(&d1_full, ci & 1, status)) break;
                    tc_fence_after();
                    float dv[32];
#pragma unroll
                    for (int tb = 0; tb < 2; ++tb) {
                        tmem_ld_16x256b_x2(lane_base + C::d1col(ci) + tk0 + 16 * tb, dv + 16 * tb);
                        tmem_ld_16x256b_x2(lane_base + (16u << 16) + C::d1col(ci) + tk0 + 16 * tb, dv + 16 * tb + 8);
                    }
                    tmem_wait_ld_regs<32>(dv);
#pragma unroll
                    for (int tb = 0; tb < 2; ++tb)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            uint32_t pf[4];
#pragma unroll
                            for (int m = 0; m < 4; ++m) {   // m = 2 bb + vh
                                const float2 u = bf2_to_f2(uf[tb][hh][m]);
                                const int e = 16 * tb + 8 * hh + 4 * (m >> 1) + 2 * (m & 1);
                                pf[m] = pack_bf16x2(u.x + dv[e], u.y + dv[e + 1]);
                            }
                            const int v = 32 * qw + 16 * hh + 8 * (mj & 1) + mr;
                            stsm_x4(smem_u32(sm + C::UOP + v * 128 + (((((tk0 + 16 * tb) >> 3) + (mj >> 1)) ^ (v & 7)) << 4)), pf);
                        }
                    tc_fence_before();
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&up_ready);
                }
            } else if (qw < 2) {   // U' = U - W S: U row i from the stage, -W S from D1 rows 0..63
                uint4 ur[NCW / 8];
#pragma unroll
                for (int e8 = 0; e8 < NCW / 8; ++e8) {
                    const int col = ucol + 8 * e8;
                    ur[e8] = trans ? make_uint4(0u, 0u, 0u, 0u)
                                   : *reinterpret_cast<const uint4*>(sb + C::U + (col >> 6) * 8192 + i * 128 +
                                                                     ((((col & 63) >> 3) ^ (i & 7)) << 4));
                }
                if (!mbar_wait(&d1_full, ci & 1, status)) break;
                tc_fence_after();
                float vv[NCW];   // D1 row i, columns jw .. jw + NCW: all loads in flight, one wait
#pragma unroll
                for (int cb = 0; cb < NCW; cb += 16)
                    tmem_ld16(lane_base + C::d1col(ci) + jw + cb, *reinterpret_cast<float(*)[16]>(vv + cb));
                tmem_wait_ld_regs<NCW>(vv);
#pragma unroll
                for (int e8 = 0; e8 < NCW / 8; ++e8) {
                    const int cc = jw / 8 + e8;   // 8-column chunk within the slice
                    float u8[8];
                    unpack8(ur[e8], u8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) u8[e] += vv[8 * e8 + e];
                    *reinterpret_cast<uint4*>(sm + C::UOP + sw128_mn_offset(8 * cc, i, C::U_LBO)) = pack8(u8);
                }
                tc_fence_before();
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&up_ready);
            }
            if (!mbar_wait(&d2_full, ci & 1, status)) break;
            tc_fence_after();
            {   // S = diag(gamma_C) S + D2 (transposed path: S^T = S^T diag(gamma_C) + D2^T, gamma per channel jw + e)
                float vv[NCW];
#pragma unroll
                for (int cb = 0; cb < NCW; cb += 16)
                    tmem_ld16(lane_base + DVS + jw + cb, *reinterpret_cast<float(*)[16]>(vv + cb));
                float gm[C::TR ? NCW : 1];
                if constexpr (C::TR) {
#pragma unroll
                    for (int e = 0; e < NCW / 4; ++e) {
                        const float4 g4 = *reinterpret_cast<const float4*>(sb + C::G + (jw + 4 * e) * 4);
                        gm[4 * e] = g4.x; gm[4 * e + 1] = g4.y; gm[4 * e + 2] = g4.z; gm[4 * e + 3] = g4.w;
                    }
                } else {
                    gm[0] = *reinterpret_cast<const float*>(sb + C::G + i * 4);
                }
                tmem_wait_ld_regs<NCW>(vv);
#pragma unroll
                for (int e = 0; e < NCW; e += 2) {
                    const float2 g2 = C::TR ? make_float2(gm[C::TR ? e : 0], gm[C::TR ? e + 1 : 0]) : f2(gm[0]);
                    const float2 a = __ffma2_rn(g2, make_float2(S[e], S[e + 1]), make_float2(vv[e], vv[e + 1]));
                    S[e] = a.x; S[e + 1] = a.y;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);   // done with this stage
            write_sop();
            tc_fence_before();
            if constexpr (!C::TR) fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_ready);
            if (C::TR && !trans && w >= NEW / 2) {
                // O^T: D1^T columns 64 + tk0 .. + 32, read while the next product 1 runs; matrix stores that
                // transpose put O's token rows into OST, which leaves by tensor stores (whole chunks) or by
                // 16-byte stores of its first n rows
                if (!mbar_wait(&o_full, ci & 1, status)) break;
                tc_fence_after();
                float dv[32];
#pragma unroll
                for (int tb = 0; tb < 2; ++tb) {
                    tmem_ld_16x256b_x2(lane_base + C::d1col(ci) + 64 + tk0 + 16 * tb, dv + 16 * tb);
                    tmem_ld_16x256b_x2(lane_base + (16u << 16) + C::d1col(ci) + 64 + tk0 + 16 * tb, dv + 16 * tb + 8);
                }
                tmem_wait_ld_regs<32>(dv);
                tc_fence_before();
                uint32_t pf[2][2][4];
#pragma unroll
                for (int tb = 0; tb < 2; ++tb)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            const int e = 16 * tb + 8 * hh + 4 * (m >> 1) + 2 * (m & 1);
                            pf[tb][hh][m] = pack_bf16x2(dv[e], dv[e + 1]);
                        }
                if (o_issuer) bulk_wait_read0();   // the previous tile has left OST
                named_bar_sync(2, 32 * NEW / 2);
                {
                    const int mj = lane >> 3, mr = lane & 7;
#pragma unroll
                    for (int tb = 0; tb < 2; ++tb)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int v0 = 32 * qw + 16 * hh + 8 * (mj & 1), tok = tk0 + 16 * tb + 8 * (mj >> 1) + mr;
                            stsm_x4_trans(smem_u32(sm + C::OST + (v0 >> 6) * 8192 + tok * 128 +
                                                   ((((v0 & 63) >> 3) ^ (tok & 7)) << 4)),
                                          pf[tb][hh]);
                        }
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 32 * NEW / 2);   // every O warp has written its part of the tile
                if (full_tma) {
                    if (o_issuer) {
#pragma unroll
                        for (int b = 0; b < DVS / 64; ++b)
                            tma_store_3d(&map_o, j0 + 64 * b, h, static_cast<int>(seq_tok0 + c * 64), sm + C::OST + b * 8192);
                        bulk_commit();
                    }
                } else {   // a ragged last chunk: rows r < n, 16 bytes (8 columns) per store
                    for (int e = t - 32 * NEW / 2; e < 64 * (DVS / 8); e += 32 * NEW / 2) {
                        const int r = e / (DVS / 8), v0 = 8 * (e % (DVS / 8));
                        if (r < n)
                            *reinterpret_cast<uint4*>(o + (static_cast<size_t>(seq_tok0 + c * 64 + r) * H + h) * DV + j0 + v0) =
                                *reinterpret_cast<const uint4*>(sm + C::OST + (v0 >> 6) * 8192 + r * 128 +
                                                                ((((v0 & 63) >> 3) ^ (r & 7)) << 4));
                    }
                }
            } else if (!C::TR && qw >= 2 && !trans) {   // O = Q gamma S + Aqk U': D1 rows 64..127, read while the next product 1 runs
                if (!mbar_wait(&o_full, ci & 1, status)) break;
                tc_fence_after();
                float vv[NCW];
#pragma unroll
                for (int cb = 0; cb < NCW; cb += 16)
                    tmem_ld16(lane_base + C::d1col(ci) + jw + cb, *reinterpret_cast<float(*)[16]>(vv + cb));
                tmem_wait_ld_regs<NCW>(vv);
                tc_fence_before();
                const int r = i - 64;   // token row
                if (full_tma) {
                    if (o_issuer) bulk_wait_read0();   // the previous tile has left OST
                    named_bar_sync(2, 32 * NEW / 2);
#pragma unroll
                    for (int e8 = 0; e8 < NCW / 8; ++e8) {
                        const int col = jw + 8 * e8;   // column within the slice
                        float o8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) o8[e] = vv[8 * e8 + e];
                        *reinterpret_cast<uint4*>(sm + C::OST + (col >> 6) * 8192 + r * 128 +
                                                  ((((col & 63) >> 3) ^ (r & 7)) << 4)) = pack8(o8);
                    }
                    fence_proxy_async_smem();
                    named_bar_sync(1, 32 * NEW / 2);   // every O warp has written its rows of the tile
                    if (o_issuer) {
#pragma unroll
                        for (int b = 0; b < DVS / 64; ++b)
                            tma_store_3d(&map_o, j0 + 64 * b, h, static_cast<int>(seq_tok0 + c * 64), sm + C::OST + b * 8192);
                        bulk_commit();
                    }
                } else if (r < n) {   // NCW columns (a multiple of 16) of row r as 16-byte stores
                    __nv_bfloat16* orow = o + (static_cast<size_t>(seq_tok0 + c * 64 + r) * H + h) * DV + j0 + jw;
#pragma unroll
                    for (int e8 = 0; e8 < NCW / 8; ++e8) {
                        float o8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) o8[e] = vv[8 * e8 + e];
                        reinterpret_cast<uint4*>(orow)[e8] = pack8(o8);
                    }
                }
            }
            // the checkpoint leaves from registers after the next product has been released, so its
            // stores drain while product 1 of the next chunk runs
            if (cpe > 0 && --ck_wait == 0) {   // chunk c ends at a multiple of ckpt_stride tokens
                ck_wait = cpe;
                if (n == 64) {
                    if (ck_slot < ck_end) {
                        float* ck = checkpoints + (static_cast<size_t>(ck_slot) * H + h) * kDK * DV + j0;
                        if constexpr (C::TR) {   // one 128-byte row segment per element index and warp
#pragma unroll
                            for (int e = 0; e < NCW; ++e) ck[srow(e) * DV + scol(e)] = S[e];
                        } else {
                            float4* dst = reinterpret_cast<float4*>(ck + i * DV + jw);
#pragma unroll
                            for (int e = 0; e < NCW / 4; ++e)
                                dst[e] = make_float4(S[4 * e], S[4 * e + 1], S[4 * e + 2], S[4 * e + 3]);
                        }
                    } else if (lane == 0) {
                        set_status(status, KDA_ERR_DEVICE_INPUT);
                    }
                }
                ++ck_slot;
            }
        }
        if (o_issuer) bulk_wait0();
        // the state (or transition) rows of this slice: pitch is the row length of the destination
        float* dst = nullptr;
        size_t pitch = 0;
        if (last) {
            if (trans) { dst = final_transition + sh * kDK * kDK + j0; pitch = kDK; }
            else if (final_state) { dst = final_state + sh * kDK * DV + j0; pitch = DV; }
        } else {
            dst = carry + sh * kDK * CW + (trans ? DV : 0) + j0;
            pitch = CW;
        }
        if (dst) {
            if constexpr (C::TR) {   // element e of every lane: one 128-byte row segment per warp
#pragma unroll
                for (int e = 0; e < NCW; ++e) dst[srow(e) * pitch + scol(e)] = S[e];
            } else {   // row i, columns jw .. + NCW: 16-byte stores (row starts and column offsets are multiples of 4)
#pragma unroll
                for (int e = 0; e < NCW / 4; ++e)
                    reinterpret_cast<float4*>(dst + i * pitch + jw)[e] =
                        make_float4(S[4 * e], S[4 * e + 1], S[4 * e + 2], S[4 * e + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tm, C::TMEM_COLS);
}

// Per window chunk: {first token, valid tokens} (n = 0 past the last chunk), so that the prep
// kernel finds any item with one load instead of a search.
__global__ void chunk_table_kernel(const int32_t* __restrict__ cu_chunks, const int32_t* __restrict__ cu_seqlens,
                                   int n_seqs, long long win_lo, long long win_hi, int2* __restrict__ tab) {
    grid_dependency_wait();   // the chunk index comes from the launch before this one
    const long long gc = win_lo + static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gc >= win_hi) return;
    ChunkLoc loc;
    tab[gc - win_lo] = locate_chunk(cu_chunks, cu_seqlens, n_seqs, gc, loc)
                           ? make_int2(static_cast<int>(loc.tok0), loc.n) : make_int2(0, 0);
}

// ------------------------------------------------------------------------------------------------
// host side
// 3D map over a [T, H, d] tensor (d innermost), box {box_d, 1, 64 tokens}, no swizzle.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int d, int H, long long T,
              int box_d, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esize, static_cast<cuuint64_t>(H) * d * esize};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_d), 1u, 64u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch with programmatic stream serialization: the kernel's blocks may be scheduled while the
// previous kernel of the stream drains, do their private set-up, and wait (grid_dependency_wait)
// before touching anything an earlier launch produced.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

template <int DV, int DVS>
cudaError_t launch_state(const ChunkArgs& a, cudaStream_t s) {
    using C = SCfg<DV, DVS>;
    const int smem = static_cast<int>(C::BYTES) + 1024;
    cudaError_t e = cudaFuncSetAttribute(state_bf16_kernel<DV, DVS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int slices = DV / DVS + (a.final_transition ? kDK / DVS : 0);
    dim3 grid(a.n_seqs * a.H, slices);
    CUtensorMap mo;   // o [T, H, DV]: 64-column x 64-token boxes with the 128-byte swizzle
    memset(&mo, 0, sizeof(mo));
    if (a.total_tokens > 0 &&
        !make_map(&mo, a.o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DV, a.H, a.total_tokens, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    return launch_pdl(state_bf16_kernel<DV, DVS>, grid, dim3(C::NT), smem, s, static_cast<const uint8_t*>(a.packets),
                      a.cu_seqlens, a.cu_chunks, a.n_seqs, a.H, a.win_lo, a.win_hi, a.initial_state,
                      static_cast<__nv_bfloat16*>(a.o), mo, a.final_state, a.final_transition, a.ckpt_stride,
                      a.checkpoints, a.ckpt_cu, a.carry, a.status);
}

template <int DV, bool MX>
cudaError_t launch_prep(const ChunkArgs& a, long long items, cudaStream_t s) {
    CUtensorMap mq, mk, mv, ml;
    const CUtensorMapDataType dt = MX ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int es = MX ? 1 : 2;
    // q, k: 64-channel half-tiles staged by TMA for the column pass (MXFP8 v codes are read with plain loads).
    // bf16 v is loaded as product B's operand: 64-column x 64-token boxes with the 128-byte swizzle, the
    // MN-major layout of the tensor-core descriptor.  log_alpha is read with plain loads (its map is unused).
    if (!make_map(&mq, a.q, dt, es, kDK, a.H, a.total_tokens, 64) ||
        !make_map(&mk, a.k, dt, es, kDK, a.H, a.total_tokens, 64) ||
        !make_map(&mv, a.v, dt, es, DV, a.H, a.total_tokens, MX ? DV : 64,
                  MX ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&ml, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kDK, a.H, a.total_tokens, 32))
        return cudaErrorInvalidValue;
    const int smem = static_cast<int>(MX ? ps::BYTES_MX : ps::BYTES) + 1024;
    cudaError_t e = cudaFuncSetAttribute(prep_bf16_kernel<DV, MX>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // all of the SM's unified L1 / shared storage as shared memory, so that two CTAs fit side by side
    e = cudaFuncSetAttribute(prep_bf16_kernel<DV, MX>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const long long slots = 2LL * num_sms();   // two CTAs per SM
    const long long grid = items < slots ? items : slots;
    return launch_pdl(prep_bf16_kernel<DV, MX>, dim3(static_cast<unsigned>(grid)), dim3(ps::NT), smem, s, mq, mk, mv,
                      ml, static_cast<const uint8_t*>(a.q), static_cast<const uint8_t*>(a.k),
                      static_cast<const uint8_t*>(a.v), a.log_alpha, a.beta, static_cast<const uint8_t*>(a.q_scale),
                      static_cast<const uint8_t*>(a.k_scale), static_cast<const uint8_t*>(a.v_scale), a.chunk_tab,
                      a.H, items, static_cast<uint8_t*>(a.packets), a.status);
}

template <int DV>
cudaError_t launch_bf16_t(const ChunkArgs& a, cudaStream_t s) {
    const long long items = (a.win_hi - a.win_lo) * a.H;
    if (a.events) cudaEventRecord(a.events->ev[1], s);
    if (a.total_tokens > 0 && items > 0) {
        const long long wchunks = a.win_hi - a.win_lo;
        cudaError_t e = launch_pdl(chunk_table_kernel, dim3(static_cast<unsigned>((wchunks + 255) / 256)), dim3(256),
                                   0, s, a.cu_chunks, a.cu_seqlens, a.n_seqs, a.win_lo, a.win_hi, a.chunk_tab);
        if (e != cudaSuccess) return e;
        e = a.mx ? launch_prep<DV, true>(a, items, s) : launch_prep<DV, false>(a, items, s);
        if (e != cudaSuccess) return e;
    }
    if (a.events) cudaEventRecord(a.events->ev[2], s);
    // dv slice per state CTA: as wide as possible while the (sequence, head) chains fill the GPU
    const long long chains = static_cast<long long>(a.n_seqs) * a.H;
    const int sms = num_sms();
    cudaError_t e;
    if (DV == 128 && chains >= (sms * 3) / 4) e = launch_state<DV, DV>(a, s);
    else if (chains * (DV / 64) >= (sms * 3) / 4) e = launch_state<DV, 64>(a, s);
    else e = launch_state<DV, 32>(a, s);
    if (a.events) cudaEventRecord(a.events->ev[3], s);
    return e;
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, []() {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

size_t chunk_packet_bytes_bf16(int dk, int dv) { return dv == 64 ? Pk<64>::BYTES : Pk<128>::BYTES; }

cudaError_t launch_chunk_bf16(const ChunkArgs& a, cudaStream_t s) {
    if (a.dk != kDK) return cudaErrorInvalidValue;
    return a.dv == 64 ? launch_bf16_t<64>(a, s) : launch_bf16_t<128>(a, s);
}

}  // namespace kda
