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
    static constexpr int R0 = (64 * DK > 2 * 64 * 64) ? 64 * DK : 2 * 64 * 64;   // g, later A + Aqk
    static constexpr int KIV = 64 * (DK > DV ? DK : DV);                          // k*Einv, later beta*V
    static constexpr size_t FLOATS = R0 + 3 * 64 * DK + KIV + 64 * 64 /*X*/ + 64 /*beta*/ + 4 * DK /*e^b*/ +
                                     4 * DK /*e^(gC-b')*/ + 16 * DK /*tile pair*/ + 3 * 256 /*solve tmp*/;
    static constexpr size_t BYTES = FLOATS * 4;
};

template <int DK, int DV>
__global__ void __launch_bounds__(256)
chunk_prep_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                      const float* __restrict__ log_alpha, const float* __restrict__ beta,
                      const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ cu_chunks, int n_seqs,
                      int H, long long win_lo, float* __restrict__ packets) {
    using P = F32Packet<DK, DV>;
    using SM = PrepSmem<DK, DV>;
    extern __shared__ __align__(16) float sm[];
    float* g = sm;                          // [64][DK]
    float* Am = sm;                         // [64][64]   (after g is dead)
    float* Aq = sm + 64 * 64;               // [64][64]
    float* KE = sm + SM::R0;                // [64][DK]   k * exp(g - b_t)
    float* QE = KE + 64 * DK;               // [64][DK]   q * exp(g - b_t)
    float* KF = QE + 64 * DK;               // [64][DK]   k * exp(b_{t+1} - g)
    float* KI = KF + 64 * DK;               // [64][DK]   k * exp(b_t - g); later beta*V [64][DV]
    float* X = KI + SM::KIV;                // [64][64]
    float* bet = X + 64 * 64;               // [64]
    float* eb = bet + 64;                   // [4][DK]    exp(b_t)
    float* ec = eb + 4 * DK;                // [4][DK]    exp(g_C - b_{t+1})
    float* ed = ec + 4 * DK;                // [4][4][DK] exp(b_i - b_jp), 1 <= jp <= i <= 3
    float* tmp = ed + 16 * DK;              // [3][16][16] solve temporaries

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
    if (t < DK) {
        float acc = 0.f;
        for (int r = 0; r < 64; ++r) { acc += g[r * DK + t]; g[r * DK + t] = acc; }
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
        KE[e] = kv * E;
        QE[e] = qv * E;
        KI[e] = kv * Einv;
        KF[e] = kv * F;
        pk[P::QT + e] = qv * E * eb[tl * DK + c];     // q * exp(g)
        pk[P::KD + e] = kv * F * ec[tl * DK + c];     // k * exp(g_C - g)
    }
    __syncthreads();   // g is dead from here; its space becomes A and Aqk
    // 4. A (strict lower, beta rows) and Aqk (inclusive lower)
    {
        const int lane = t & 31, w = t >> 5;
        for (int rr = 0; rr < 8; ++rr) {
            const int r = w + 8 * rr, ti = r >> 4;
            for (int half = 0; half < 2; ++half) {
                const int s = lane + 32 * half, tj = s >> 4;
                float ak = 0.f, aq = 0.f;
                if (s <= r) {
                    if (tj == ti) {
                        for (int cc = 0; cc < DK; ++cc) {
                            const int c = (cc + lane) & (DK - 1);
                            const float kr = KI[s * DK + c];
                            ak = fmaf(KE[r * DK + c], kr, ak);
                            aq = fmaf(QE[r * DK + c], kr, aq);
                        }
                    } else {
                        const float* d = ed + (ti * 4 + tj + 1) * DK;
                        for (int cc = 0; cc < DK; ++cc) {
                            const int c = (cc + lane) & (DK - 1);
                            const float kr = KF[s * DK + c] * d[c];
                            ak = fmaf(KE[r * DK + c], kr, ak);
                            aq = fmaf(QE[r * DK + c], kr, aq);
                        }
                    }
                }
                Am[r * 64 + s] = s < r ? bet[r] * ak : 0.f;
                Aq[r * 64 + s] = aq;
            }
        }
    }
    __syncthreads();
    for (int e = t; e < 64 * 64; e += 256) pk[P::AQ + e] = Aq[e];
    // stage beta * V over KI (dead) and beta * k * exp(g) over KE (dead)
    for (int e = t; e < 64 * DV; e += 256) {
        const int r = e / DV, c = e % DV;
        KI[e] = r < n ? bet[r] * vb[static_cast<size_t>(r) * row_v + c] : 0.f;
    }
    for (int e = t; e < 64 * DK; e += 256) {
        const int r = e / DK, c = e % DK;
        KE[e] = bet[r] * KE[e] * eb[(r >> 4) * DK + c];
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
    // 6. W = X (beta K exp(g)),  U = X (beta V)
    for (int e = t; e < 64 * DK; e += 256) {
        const int r = e / DK, c = e % DK;
        float acc = 0.f;
        for (int s = 0; s <= r; ++s) acc = fmaf(X[r * 64 + s], KE[s * DK + c], acc);
        pk[P::W + e] = acc;
    }
    for (int e = t; e < 64 * DV; e += 256) {
        const int r = e / DV, c = e % DV;
        float acc = 0.f;
        for (int s = 0; s <= r; ++s) acc = fmaf(X[r * 64 + s], KI[s * DV + c], acc);
        pk[P::U + e] = acc;
    }
}

constexpr int kF32Cols = 32;   // dv columns per state CTA

template <int DK, int DV>
struct StateSmem {
    static constexpr size_t FLOATS = DK * kF32Cols /*S*/ + 3 * 64 * DK /*W,QT,KD*/ + 2 * 64 * kF32Cols /*U,U'*/ +
                                     64 * 64 /*Aqk*/ + DK /*G*/;
    static constexpr size_t BYTES = FLOATS * 4;
};

// One CTA per (sequence, head, 32-column slice).  Slices [0, DV/32) are state columns; with a
// transition output, slices [DV/32, DV/32 + DK/32) carry columns of the cumulative transition
// (same update with U = 0, identity start, no output).
template <int DK, int DV>
__global__ void __launch_bounds__(256)
chunk_state_f32_kernel(const float* __restrict__ packets, const int32_t* __restrict__ cu_seqlens,
                       const int32_t* __restrict__ cu_chunks, int n_seqs, int H, long long win_lo,
                       long long win_hi, bool multi_window, const float* __restrict__ initial_state,
                       float* __restrict__ o, float* __restrict__ final_state, float* __restrict__ final_transition,
                       int ckpt_stride, float* __restrict__ checkpoints, const int32_t* __restrict__ ckpt_cu,
                       float* __restrict__ carry, int* status) {
    using P = F32Packet<DK, DV>;
    constexpr int NC = kF32Cols;
    extern __shared__ __align__(16) float sm[];
    float* S = sm;                 // [DK][NC]
    float* Wc = S + DK * NC;       // [64][DK]
    float* Qc = Wc + 64 * DK;      // [64][DK]
    float* Kc = Qc + 64 * DK;      // [64][DK]
    float* Uc = Kc + 64 * DK;      // [64][NC]
    float* Up = Uc + 64 * NC;      // [64][NC]
    float* Ac = Up + 64 * NC;      // [64][64]
    float* Gc = Ac + 64 * 64;      // [DK]

    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
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

    // initial state slice
    for (int e = t; e < DK * NC; e += 256) {
        const int i = e / NC, j = e % NC;
        float x;
        if (!first) x = carry[(sh * DK + i) * CW + (trans ? DV : 0) + c0 + j];
        else if (trans) x = (i == c0 + j) ? 1.f : 0.f;
        else x = initial_state ? initial_state[(sh * DK + i) * DV + c0 + j] : 0.f;
        S[e] = x;
    }
    __syncthreads();
    const long long seq_tok0 = cu_seqlens[seq];
    const long long seq_len = static_cast<long long>(cu_seqlens[seq + 1]) - seq_tok0;
    for (long long gcix = lo; gcix < hi; ++gcix) {
        const int c = static_cast<int>(gcix - ch_lo);
        const long long rem = seq_len - static_cast<long long>(c) * 64;
        const int n = rem < 64 ? static_cast<int>(rem) : 64;
        const float* pk = packets + static_cast<size_t>((gcix - win_lo) * H + h) * (P::BYTES / 4);
        for (int e = t; e < 64 * DK; e += 256) {
            Wc[e] = pk[P::W + e];
            Qc[e] = pk[P::QT + e];
            Kc[e] = pk[P::KD + e];
        }
        for (int e = t; e < 64 * NC; e += 256) {
            const int r = e / NC, j = e % NC;
            Uc[e] = trans ? 0.f : pk[P::U + r * DV + c0 + j];
        }
        for (int e = t; e < 64 * 64; e += 256) Ac[e] = pk[P::AQ + e];
        for (int e = t; e < DK; e += 256) Gc[e] = pk[P::G + e];
        __syncthreads();
        // U' = U - W S
        for (int m = 0; m < 8; ++m) {
            const int r = w + 8 * m;
            float acc = Uc[r * NC + lane];
            for (int i = 0; i < DK; ++i) acc = fmaf(-Wc[r * DK + i], S[i * NC + lane], acc);
            Up[r * NC + lane] = acc;
        }
        __syncthreads();
        // O = Qt S + Aqk U'
        if (!trans) {
            for (int m = 0; m < 8; ++m) {
                const int r = w + 8 * m;
                if (r >= n) continue;
                float acc = 0.f;
                for (int i = 0; i < DK; ++i) acc = fmaf(Qc[r * DK + i], S[i * NC + lane], acc);
                for (int s = 0; s <= r; ++s) acc = fmaf(Ac[r * 64 + s], Up[s * NC + lane], acc);
                o[(static_cast<size_t>(seq_tok0 + c * 64 + r) * H + h) * DV + c0 + lane] = acc;
            }
        }
        __syncthreads();
        // S <- Diag(exp(g_C)) S + Kdec^T U'
        for (int m = 0; m < DK / 8; ++m) {
            const int i = w + 8 * m;
            float acc = Gc[i] * S[i * NC + lane];
            for (int r = 0; r < 64; ++r) acc = fmaf(Kc[r * DK + i], Up[r * NC + lane], acc);
            S[i * NC + lane] = acc;
        }
        __syncthreads();
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
