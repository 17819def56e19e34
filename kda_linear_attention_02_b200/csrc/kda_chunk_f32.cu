// kda_chunk_f32.cu -- chunked KDA forward for fp32 inputs (SIMT fp32 throughout).
//
// The precision path: fp32 q/k/v with a 1e-4 relative error budget, which bf16 tensor-core
// operands (unit roundoff 2^-9) cannot meet.  It computes the same chunk algebra as the bf16
// tcgen05 path, with fp32 FMA:
//
// Per chunk of C = 64 tokens (positions r), lambda = max(log_alpha, ln 0.0067) (orkas.ai "Kimi K3
// architecture" post, decay-floor section), g = chunk-local inclusive cumsum of lambda, b_t = g just
// before 16-token tile t (0 for the first tile), and
//   A[r,s]   = beta_r sum_c k_rc k_sc exp(g_rc - g_sc)   (s < r)          -- "(I + strict_tril(..))"
//   Aqk[r,s] = sum_c q_rc k_sc exp(g_rc - g_sc)          (s <= r)
//   X = (I + A)^-1 by blocked forward substitution over 16 x 16 tiles
//   W = X diag(beta) (K * exp(g)),  U = X diag(beta) V
// then, sequentially over chunks with the state S (fp32):
//   U' = U - W S;  O = (Q * exp(g)) S + Aqk U';  S <- Diag(exp(g_C)) S + (K * exp(g_C - g))^T U'.
//
// exp(g_r - g_s) is never formed per pair.  Each factor is split at a tile anchor so that no factor
// leaves the fp32 range: inside one tile exp(b_t - g_s) <= exp(-16 ln 0.0067) = e^80.09 (the
// decay-floor bound of the orkas.ai post), across tiles both factors are <= 1.
//   same tile t:        exp(g_r - b_t) * exp(b_t - g_s)
//   row tile i > j:     exp(g_r - b_i) * exp(b_i - b_{j+1}) * exp(b_{j+1} - g_s)
#include "kda_chunk_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

template <int DK, int DV>
struct F32Packet {
    // float offsets inside one (chunk, head) packet
    static constexpr size_t W = 0;                      // [64][DK]
    static constexpr size_t U = W + 64 * DK;            // [64][DV]
    static constexpr size_t QT = U + 64 * DV;           // [64][DK]  q * exp(g)
    static constexpr size_t KD = QT + 64 * DK;          // [64][DK]  k * exp(g_C - g)
    static constexpr size_t AQ = KD + 64 * DK;          // [64][64]
    static constexpr size_t G = AQ + 64 * 64;           // [DK]      exp(g_C)
    static constexpr size_t FLOATS = G + DK;
    static constexpr size_t BYTES = ((FLOATS * 4 + 255) / 256) * 256;
};

template <int DK, int DV>
struct PrepSmem {
    static constexpr int TP = 64 + 4;   // pitch of the transposed factor arrays [DK][TP] (float4 rows of 4 tokens)
    static constexpr int R0 = (64 * DK > 2 * 64 * 64) ? 64 * DK : 2 * 64 * 64;   // g, later A + Aqk
    static constexpr int FT = DK * TP;                                             // one transposed factor array
    static constexpr int KIV = FT > 64 * DV ? FT : 64 * DV;                        // k*Einv^T, later beta*V
    static constexpr size_t FLOATS = R0 + 3 * FT + KIV + 64 * 64 /*X*/ + 64 /*beta*/ + 4 * DK /*e^b*/ +
                                     4 * DK /*e^(gC-b')*/ + 16 * DK /*tile pair*/ + 3 * 256 /*solve tmp*/;
    static constexpr size_t BYTES = FLOATS * 4;
};

// One CTA per (chunk, head) item.  The elementwise factors are stored transposed (channel-major, 4 tokens
// per float4), so that the A / Aqk products, W and U run as 4 x 4 (or 4 x 8) register blocks per thread.
template <int DK, int DV>
__global__ void __launch_bounds__(256)
chunk_prep_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                      const float* __restrict__ log_alpha, const float* __restrict__ beta,
                      const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ cu_chunks, int n_seqs,
                      int H, long long win_lo, float* __restrict__ packets) {
    using P = F32Packet<DK, DV>;
    using SM = PrepSmem<DK, DV>;
    constexpr int TP = SM::TP;
    extern __shared__ __align__(16) float sm[];
    float* g = sm;                          // [64][DK]
    float* Am = sm;                         // [64][64]   (after g is dead)
    float* Aq = sm + 64 * 64;               // [64][64]
    float* KE = sm + SM::R0;                // [DK][TP]   k * exp(g - b_t), transposed; later beta k gamma [64][DK]
    float* QE = KE + SM::FT;                // [DK][TP]   q * exp(g - b_t), transposed
    float* KF = QE + SM::FT;                // [DK][TP]   k * exp(b_{t+1} - g), transposed
    float* KI = KF + SM::FT;                // [DK][TP]   k * exp(b_t - g), transposed; later beta*V [64][DV]
    float* BK = QE;                         // [64][DK]   beta k gamma (QE is dead by then)
    float* X = KI + SM::KIV;                // [64][64]
    float* bet = X + 64 * 64;               // [64]
    float* eb = bet + 64;                   // [4][DK]    exp(b_t)
    float* ec = eb + 4 * DK;                // [4][DK]    exp(g_C - b_{t+1})
    float* ed = ec + 4 * DK;                // [4][4][DK] exp(b_i - b_jp), 1 <= jp <= i <= 3
    float* tmp = ed + 16 * DK;              // [3][16][16] solve temporaries; the prefix sum's segment totals

    const int t = threadIdx.x;
    const long long item = blockIdx.x;
    const long long gc = win_lo + item / H;
    const int h = static_cast<int>(item % H);
    ChunkLoc loc;
    if (!locate_chunk(cu_chunks, cu_seqlens, n_seqs, gc, loc)) return;
    float* pk = packets + static_cast<size_t>(item) * (P::BYTES / 4);
    const int n = loc.n;
    const size_t row_k = static_cast<size_t>(H) * DK, row_v = static_cast<size_t>(H) * DV;
    const float* qb = q + static_cast<size_t>(loc.tok0) * row_k + static_cast<size_t>(h) * DK;
    const float* kb = k + static_cast<size_t>(loc.tok0) * row_k + static_cast<size_t>(h) * DK;
    const float* vb = v + static_cast<size_t>(loc.tok0) * row_v + static_cast<size_t>(h) * DV;
    const float* lb = log_alpha + static_cast<size_t>(loc.tok0) * row_k + static_cast<size_t>(h) * DK;

    // 1. floored log-decay, chunk-local inclusive cumsum (padded rows: lambda = 0, beta = 0)
    for (int e = t; e < 64 * DK; e += 256) {
        const int r = e / DK, c = e % DK;
        g[e] = r < n ? floor_log_decay(lb[static_cast<size_t>(r) * row_k + c]) : 0.f;
    }
    if (t < 64) bet[t] = t < n ? beta[(static_cast<size_t>(loc.tok0) + t) * H + h] : 0.f;
    __syncthreads();
    {   // inclusive prefix sum along the 64 tokens: 256 / DK segments per channel, then the segments' offsets
        constexpr int NSEG = 256 / DK, LSEG = 64 / NSEG;
        const int c = t % DK, sg = t / DK;
        float acc = 0.f;
        for (int r = sg * LSEG; r < (sg + 1) * LSEG; ++r) { acc += g[r * DK + c]; g[r * DK + c] = acc; }
        tmp[sg * DK + c] = acc;
        __syncthreads();
        float off = 0.f;
        for (int s2 = 0; s2 < sg; ++s2) off += tmp[s2 * DK + c];
        if (sg > 0)
            for (int r = sg * LSEG; r < (sg + 1) * LSEG; ++r) g[r * DK + c] += off;
    }
    __syncthreads();
    // 2. per-(tile, channel) factors
    if (t < DK) {
        float b[5];
        b[0] = 0.f;
        for (int i = 1; i <= 4; ++i) b[i] = g[(16 * i - 1) * DK + t];   // b[4] = g_C
        for (int i = 0; i < 4; ++i) { eb[i * DK + t] = expf(b[i]); ec[i * DK + t] = expf(b[4] - b[i + 1]); }
        for (int i = 1; i < 4; ++i)
            for (int jp = 1; jp <= i; ++jp) ed[(i * 4 + jp) * DK + t] = expf(b[i] - b[jp]);
        pk[P::G + t] = expf(b[4]);
    }
    __syncthreads();
    // 3. anchored elementwise factors
    for (int e = t; e < 64 * DK; e += 256) {
        const int r = e / DK, c = e % DK, tl = r >> 4;
        const float bt = tl ? g[(16 * tl - 1) * DK + c] : 0.f;
        const float bn = g[(16 * tl + 15) * DK + c];
        const float gr = g[e];
        const float kv = r < n ? kb[static_cast<size_t>(r) * row_k + c] : 0.f;
        const float qv = r < n ? qb[static_cast<size_t>(r) * row_k + c] : 0.f;
        const float E = expf(gr - bt), Einv = expf(bt - gr), F = expf(bn - gr);
        KE[c * TP + r] = kv * E;
        QE[c * TP + r] = qv * E;
        KI[c * TP + r] = kv * Einv;
        KF[c * TP + r] = kv * F;
        pk[P::QT + e] = qv * E * eb[tl * DK + c];     // q * exp(g)
        pk[P::KD + e] = kv * F * ec[tl * DK + c];     // k * exp(g_C - g)
    }
    __syncthreads();   // g is dead from here; its space becomes A and Aqk
    // 4. A (strict lower, beta rows) and Aqk (inclusive lower): thread = 4 x 4 block (rows r0.., keys s0..);
    //    both lie in one 16-token tile each, so the key side is one variant for the whole block
    {
        const int rb = t >> 4, sb = t & 15, r0 = 4 * rb, s0 = 4 * sb;
        float ak[4][4], aq[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int x = 0; x < 4; ++x) ak[u][x] = aq[u][x] = 0.f;
        if (sb <= rb) {   // blocks above the diagonal are zero
            const int ti = r0 >> 4, tj = s0 >> 4;
            const bool diag = ti == tj;
            const float* kside = diag ? KI : KF;
            const float* d = ed + (ti * 4 + tj + 1) * DK;   // exp(b_ti - b_{tj+1}), read off the diagonal only
            for (int c = 0; c < DK; ++c) {
                const float4 ke = *reinterpret_cast<const float4*>(KE + c * TP + r0);
                const float4 qe = *reinterpret_cast<const float4*>(QE + c * TP + r0);
                float4 kr = *reinterpret_cast<const float4*>(kside + c * TP + s0);
                if (!diag) {
                    const float dc = d[c];
                    kr = make_float4(kr.x * dc, kr.y * dc, kr.z * dc, kr.w * dc);
                }
                const float kev[4] = {ke.x, ke.y, ke.z, ke.w}, qev[4] = {qe.x, qe.y, qe.z, qe.w};
                const float krv[4] = {kr.x, kr.y, kr.z, kr.w};
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        ak[u][x] = fmaf(kev[u], krv[x], ak[u][x]);
                        aq[u][x] = fmaf(qev[u], krv[x], aq[u][x]);
                    }
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = r0 + u;
            const float br = bet[r];
            float a4[4], q4[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                a4[x] = s0 + x < r ? br * ak[u][x] : 0.f;
                q4[x] = s0 + x <= r ? aq[u][x] : 0.f;
            }
            *reinterpret_cast<float4*>(Am + r * 64 + s0) = make_float4(a4[0], a4[1], a4[2], a4[3]);
            *reinterpret_cast<float4*>(Aq + r * 64 + s0) = make_float4(q4[0], q4[1], q4[2], q4[3]);
        }
    }
    __syncthreads();
    for (int e = t; e < 64 * 64; e += 256) pk[P::AQ + e] = Aq[e];
    // stage beta * V over KI (dead) and beta * k * exp(g) over QE (dead), both row-major
    for (int e = t; e < 64 * DV; e += 256) {
        const int r = e / DV, c = e % DV;
        KI[e] = r < n ? bet[r] * vb[static_cast<size_t>(r) * row_v + c] : 0.f;
    }
    for (int e = t; e < 64 * DK; e += 256) {
        const int r = e / DK, c = e % DK;
        BK[e] = bet[r] * KE[c * TP + r] * eb[(r >> 4) * DK + c];
    }
    // 5. X = (I + A)^-1: diagonal 16x16 blocks (one warp each, lane = column), then off-diagonal
    //    blocks by block-diagonal level: X_ij = -X_ii sum_{j<=m<i} A_im X_mj
    if (t < 128) {
        const int blk = t >> 5, col = t & 31;
        if (col < 16) {
            const int o0 = blk * 16;
            for (int r = 0; r < 16; ++r) {
                float x = (r == col) ? 1.f : 0.f;
                for (int m = col; m < r; ++m) x = fmaf(-Am[(o0 + r) * 64 + o0 + m], X[(o0 + m) * 64 + o0 + col], x);
                X[(o0 + r) * 64 + o0 + col] = x;
            }
        }
    }
    for (int e = t; e < 64 * 64; e += 256) {   // zero the strictly-upper blocks
        const int r = e >> 6, s = e & 63;
        if ((s >> 4) > (r >> 4)) X[e] = 0.f;
    }
    __syncthreads();
    for (int d = 1; d < 4; ++d) {
        const int nb = 4 - d;
        for (int e = t; e < nb * 256; e += 256) {
            const int bi = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            const int i = bi + d, j = bi;
            float acc = 0.f;
            for (int m = 16 * j; m < 16 * i; ++m) acc = fmaf(Am[(16 * i + rr) * 64 + m], X[m * 64 + 16 * j + cc], acc);
            tmp[e] = acc;
        }
        __syncthreads();
        for (int e = t; e < nb * 256; e += 256) {
            const int bi = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            const int i = bi + d, j = bi;
            float acc = 0.f;
            for (int m = 0; m <= rr; ++m) acc = fmaf(X[(16 * i + rr) * 64 + 16 * i + m], tmp[bi * 256 + m * 16 + cc], acc);
            X[(16 * i + rr) * 64 + 16 * j + cc] = -acc;
        }
        __syncthreads();
    }
    // 6. W = X (beta K exp(g)),  U = X (beta V): thread = 4 rows x (DK / 16 and DV / 16) columns
    {
        constexpr int CK = DK / 16, CV = DV / 16;
        const int r0 = 4 * (t >> 4), cb = t & 15;
        float aw[4][CK], au[4][CV];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int x = 0; x < CK; ++x) aw[u][x] = 0.f;
#pragma unroll
            for (int x = 0; x < CV; ++x) au[u][x] = 0.f;
        }
        for (int s2 = 0; s2 < r0 + 4; ++s2) {   // X is zero past its diagonal
            float xr[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) xr[u] = X[(r0 + u) * 64 + s2];
#pragma unroll
            for (int x4 = 0; x4 < CK; x4 += 4) {
                const float4 b = *reinterpret_cast<const float4*>(BK + s2 * DK + cb * CK + x4);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    aw[u][x4] = fmaf(xr[u], b.x, aw[u][x4]);
                    aw[u][x4 + 1] = fmaf(xr[u], b.y, aw[u][x4 + 1]);
                    aw[u][x4 + 2] = fmaf(xr[u], b.z, aw[u][x4 + 2]);
                    aw[u][x4 + 3] = fmaf(xr[u], b.w, aw[u][x4 + 3]);
                }
            }
#pragma unroll
            for (int x4 = 0; x4 < CV; x4 += 4) {
                const float4 b = *reinterpret_cast<const float4*>(KI + s2 * DV + cb * CV + x4);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    au[u][x4] = fmaf(xr[u], b.x, au[u][x4]);
                    au[u][x4 + 1] = fmaf(xr[u], b.y, au[u][x4 + 1]);
                    au[u][x4 + 2] = fmaf(xr[u], b.z, au[u][x4 + 2]);
                    au[u][x4 + 3] = fmaf(xr[u], b.w, au[u][x4 + 3]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int x4 = 0; x4 < CK; x4 += 4)
                *reinterpret_cast<float4*>(pk + P::W + (r0 + u) * DK + cb * CK + x4) =
                    make_float4(aw[u][x4], aw[u][x4 + 1], aw[u][x4 + 2], aw[u][x4 + 3]);
#pragma unroll
            for (int x4 = 0; x4 < CV; x4 += 4)
                *reinterpret_cast<float4*>(pk + P::U + (r0 + u) * DV + cb * CV + x4) =
                    make_float4(au[u][x4], au[u][x4 + 1], au[u][x4 + 2], au[u][x4 + 3]);
        }
    }
}

constexpr int kF32Cols = 16;   // dv columns per state CTA

// Shared memory of the state pass, in floats; rows of the operands read as float4 along their K index
// are padded by 4 floats, so that the 8 rows a quarter warp reads fall on different banks.
template <int DK, int DV>
struct StateSmem {
    static constexpr int NC = kF32Cols;
    static constexpr int PK = DK + 4, PA = 64 + 4;
    static constexpr size_t S0 = 0;                    // S [DK][NC], two buffers (read one, write the other)
    static constexpr size_t W = 2 * DK * NC;           // -W rows [64][PK]
    static constexpr size_t QT = W + 64 * PK;          // Q gamma rows [64][PK]
    static constexpr size_t KD = QT + 64 * PK;         // Kdec rows [64][DK]
    static constexpr size_t AQ = KD + 64 * DK;         // Aqk rows [64][PA]
    static constexpr size_t UC = AQ + 64 * PA;         // U slice [64][NC]
    static constexpr size_t UP = UC + 64 * NC;         // U' slice [64][NC]
    static constexpr size_t G = UP + 64 * NC;          // exp(g_C) [DK]
    static constexpr size_t FLOATS = G + DK;
    static constexpr size_t BYTES = FLOATS * 4;
};

// One CTA per (sequence, head, 16-column slice).  Slices [0, DV/16) are state columns; with a
// transition output, slices [DV/16, DV/16 + DK/16) carry columns of the cumulative transition
// (same update with U = 0, identity start, no output).  Each thread forms four adjacent columns of one
// row of U', O and the new S from 16-byte shared loads, summing in the same order as a plain dot product.
template <int DK, int DV>
__global__ void __launch_bounds__(256)
chunk_state_f32_kernel(const float* __restrict__ packets, const int32_t* __restrict__ cu_seqlens,
                       const int32_t* __restrict__ cu_chunks, int n_seqs, int H, long long win_lo,
                       long long win_hi, bool multi_window, const float* __restrict__ initial_state,
                       float* __restrict__ o, float* __restrict__ final_state, float* __restrict__ final_transition,
                       int ckpt_stride, float* __restrict__ checkpoints, const int32_t* __restrict__ ckpt_cu,
                       float* __restrict__ carry, int* status) {
    using P = F32Packet<DK, DV>;
    using L = StateSmem<DK, DV>;
    constexpr int NC = kF32Cols, PK = L::PK, PA = L::PA;
    extern __shared__ __align__(16) float sm[];
    float* Wc = sm + L::W;
    float* Qc = sm + L::QT;
    float* Kc = sm + L::KD;
    float* Ac = sm + L::AQ;
    float* Uc = sm + L::UC;
    float* Up = sm + L::UP;
    float* Gc = sm + L::G;

    const int t = threadIdx.x;
    const int rr = t >> 2, cq = 4 * (t & 3);   // this thread's row (of U', O, S) and first column
    const int seq = blockIdx.x / H, h = blockIdx.x % H;
    const int slice = blockIdx.y;
    const bool trans = slice >= DV / NC;
    const int c0 = trans ? (slice - DV / NC) * NC : slice * NC;
    if (trans && !final_transition) return;
    const long long ch_lo = cu_chunks[seq], ch_hi = cu_chunks[seq + 1];
    const long long lo = ch_lo > win_lo ? ch_lo : win_lo;
    const long long hi = ch_hi < win_hi ? ch_hi : win_hi;
    const bool empty_seq = ch_lo == ch_hi;
    if (!(lo < hi) && !(empty_seq && win_lo == 0)) return;
    const bool first = empty_seq || ch_lo >= win_lo;
    const bool last = empty_seq || ch_hi <= win_hi;
    const size_t sh = static_cast<size_t>(seq) * H + h;
    const int CW = DV + DK;   // carry row width

    float* S = sm + L::S0;            // the current state slice [DK][NC]
    float* Sn = sm + L::S0 + DK * NC; // the next one
    for (int e = t; e < DK * NC; e += 256) {
        const int i = e / NC, j = e % NC;
        float x;
        if (!first) x = carry[(sh * DK + i) * CW + (trans ? DV : 0) + c0 + j];
        else if (trans) x = (i == c0 + j) ? 1.f : 0.f;
        else x = initial_state ? initial_state[(sh * DK + i) * DV + c0 + j] : 0.f;
        S[e] = x;
    }
    const long long seq_tok0 = cu_seqlens[seq];
    const long long seq_len = static_cast<long long>(cu_seqlens[seq + 1]) - seq_tok0;
    for (long long gcix = lo; gcix < hi; ++gcix) {
        const int c = static_cast<int>(gcix - ch_lo);
        const long long rem = seq_len - static_cast<long long>(c) * 64;
        const int n = rem < 64 ? static_cast<int>(rem) : 64;
        const float* pk = packets + static_cast<size_t>((gcix - win_lo) * H + h) * (P::BYTES / 4);
        // this chunk's packet (16-byte loads; every offset below is a multiple of 4 floats)
        for (int e = t; e < 64 * DK / 4; e += 256) {
            const int r = (4 * e) / DK, i = (4 * e) % DK;
            *reinterpret_cast<float4*>(Wc + r * PK + i) = reinterpret_cast<const float4*>(pk + P::W)[e];
            *reinterpret_cast<float4*>(Qc + r * PK + i) = reinterpret_cast<const float4*>(pk + P::QT)[e];
            reinterpret_cast<float4*>(Kc)[e] = reinterpret_cast<const float4*>(pk + P::KD)[e];
        }
        for (int e = t; e < 64 * 16; e += 256) {
            const int r = e >> 4, s4 = 4 * (e & 15);
            *reinterpret_cast<float4*>(Ac + r * PA + s4) = reinterpret_cast<const float4*>(pk + P::AQ)[e];
        }
        for (int e = t; e < 64 * NC / 4; e += 256) {
            const int r = (4 * e) / NC, j = (4 * e) % NC;
            reinterpret_cast<float4*>(Uc)[e] = trans ? make_float4(0.f, 0.f, 0.f, 0.f)
                                                     : *reinterpret_cast<const float4*>(pk + P::U + r * DV + c0 + j);
        }
        for (int e = t; e < DK; e += 256) Gc[e] = pk[P::G + e];
        __syncthreads();
        // U' = U - W S: row rr, columns cq .. cq + 3
        {
            float4 acc = *reinterpret_cast<const float4*>(Uc + rr * NC + cq);
            for (int i = 0; i < DK; i += 4) {
                const float4 w4 = *reinterpret_cast<const float4*>(Wc + rr * PK + i);
                const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 s4 = *reinterpret_cast<const float4*>(S + (i + u) * NC + cq);
                    acc.x = fmaf(-wv[u], s4.x, acc.x);
                    acc.y = fmaf(-wv[u], s4.y, acc.y);
                    acc.z = fmaf(-wv[u], s4.z, acc.z);
                    acc.w = fmaf(-wv[u], s4.w, acc.w);
                }
            }
            *reinterpret_cast<float4*>(Up + rr * NC + cq) = acc;
        }
        __syncthreads();
        // O = Qt S + Aqk U' (row rr) and the next state S' = Diag(exp(g_C)) S + Kdec^T U' (rows i = rr + 64 p)
        if (!trans && rr < n) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int i = 0; i < DK; i += 4) {
                const float4 q4 = *reinterpret_cast<const float4*>(Qc + rr * PK + i);
                const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 s4 = *reinterpret_cast<const float4*>(S + (i + u) * NC + cq);
                    acc.x = fmaf(qv[u], s4.x, acc.x);
                    acc.y = fmaf(qv[u], s4.y, acc.y);
                    acc.z = fmaf(qv[u], s4.z, acc.z);
                    acc.w = fmaf(qv[u], s4.w, acc.w);
                }
            }
            for (int s4i = 0; s4i <= rr; s4i += 4) {   // Aqk is zero past the diagonal
                const float4 a4 = *reinterpret_cast<const float4*>(Ac + rr * PA + s4i);
                const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (s4i + u > rr) continue;
                    const float4 p4 = *reinterpret_cast<const float4*>(Up + (s4i + u) * NC + cq);
                    acc.x = fmaf(av[u], p4.x, acc.x);
                    acc.y = fmaf(av[u], p4.y, acc.y);
                    acc.z = fmaf(av[u], p4.z, acc.z);
                    acc.w = fmaf(av[u], p4.w, acc.w);
                }
            }
            *reinterpret_cast<float4*>(o + (static_cast<size_t>(seq_tok0 + c * 64 + rr) * H + h) * DV + c0 + cq) = acc;
        }
#pragma unroll
        for (int pp = 0; pp < DK / 64; ++pp) {
            const int i = rr + 64 * pp;
            const float gi = Gc[i];
            const float4 s0 = *reinterpret_cast<const float4*>(S + i * NC + cq);
            float4 acc = make_float4(gi * s0.x, gi * s0.y, gi * s0.z, gi * s0.w);
            for (int r = 0; r < 64; ++r) {
                const float kv = Kc[r * DK + i];
                const float4 p4 = *reinterpret_cast<const float4*>(Up + r * NC + cq);
                acc.x = fmaf(kv, p4.x, acc.x);
                acc.y = fmaf(kv, p4.y, acc.y);
                acc.z = fmaf(kv, p4.z, acc.z);
                acc.w = fmaf(kv, p4.w, acc.w);
            }
            *reinterpret_cast<float4*>(Sn + i * NC + cq) = acc;
        }
        __syncthreads();   // S' complete; the packet buffers and U' free for the next chunk
        float* tmp = S; S = Sn; Sn = tmp;
        if (!trans && ckpt_stride > 0 && checkpoints && n == 64) {
            const long long end = static_cast<long long>(c + 1) * 64;
            if (end % ckpt_stride == 0) {
                const long long slot = ckpt_cu[seq] + end / ckpt_stride - 1;
                if (slot < ckpt_cu[seq] || slot >= ckpt_cu[seq + 1]) {   // table disagrees with cu_seqlens
                    if (t == 0) set_status(status, KDA_ERR_DEVICE_INPUT);
                    continue;
                }
                for (int e = t; e < DK * NC; e += 256) {
                    const int i = e / NC, j = e % NC;
                    checkpoints[((static_cast<size_t>(slot) * H + h) * DK + i) * DV + c0 + j] = S[e];
                }
            }
        }
    }
    for (int e = t; e < DK * NC; e += 256) {
        const int i = e / NC, j = e % NC;
        if (last) {
            if (trans) final_transition[(sh * DK + i) * DK + c0 + j] = S[e];
            else if (final_state) final_state[(sh * DK + i) * DV + c0 + j] = S[e];
        } else {
            carry[(sh * DK + i) * CW + (trans ? DV : 0) + c0 + j] = S[e];
        }
    }
}

template <int DK, int DV>
cudaError_t launch_f32_t(const ChunkArgs& a, cudaStream_t s) {
    using SM = PrepSmem<DK, DV>;
    using SS = StateSmem<DK, DV>;
    cudaError_t e = cudaFuncSetAttribute(chunk_prep_f32_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(SM::BYTES));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_state_f32_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(SS::BYTES));
    if (e != cudaSuccess) return e;
    const long long items = (a.win_hi - a.win_lo) * a.H;
    if (a.events) cudaEventRecord(a.events->ev[1], s);
    if (items > 0)
        chunk_prep_f32_kernel<DK, DV><<<static_cast<unsigned>(items), 256, SM::BYTES, s>>>(
            static_cast<const float*>(a.q), static_cast<const float*>(a.k), static_cast<const float*>(a.v),
            a.log_alpha, a.beta, a.cu_seqlens, a.cu_chunks, a.n_seqs, a.H, a.win_lo, static_cast<float*>(a.packets));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int slices = DV / kF32Cols + (a.final_transition ? DK / kF32Cols : 0);
    dim3 grid(a.n_seqs * a.H, slices);
    if (a.events) cudaEventRecord(a.events->ev[2], s);
    chunk_state_f32_kernel<DK, DV><<<grid, 256, SS::BYTES, s>>>(
        static_cast<const float*>(a.packets), a.cu_seqlens, a.cu_chunks, a.n_seqs, a.H, a.win_lo, a.win_hi,
        a.multi_window, a.initial_state, static_cast<float*>(a.o), a.final_state, a.final_transition, a.ckpt_stride,
        a.checkpoints, a.ckpt_cu, a.carry, a.status);
    if (a.events) cudaEventRecord(a.events->ev[3], s);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_packet_bytes_f32(int dk, int dv) {
    if (dk == 128 && dv == 128) return F32Packet<128, 128>::BYTES;
    if (dk == 128 && dv == 64) return F32Packet<128, 64>::BYTES;
    if (dk == 64 && dv == 128) return F32Packet<64, 128>::BYTES;
    return F32Packet<64, 64>::BYTES;
}

cudaError_t launch_chunk_f32(const ChunkArgs& a, cudaStream_t s) {
    if (a.dk == 128 && a.dv == 128) return launch_f32_t<128, 128>(a, s);
    if (a.dk == 128 && a.dv == 64) return launch_f32_t<128, 64>(a, s);
    if (a.dk == 64 && a.dv == 128) return launch_f32_t<64, 128>(a, s);
    return launch_f32_t<64, 64>(a, s);
}

}  // namespace kda
