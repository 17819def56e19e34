// kda_chunk_common.cuh -- indexing shared by the two chunk paths (fp32 SIMT and bf16 tcgen05).
//
// A packed batch of N sequences is cut, per sequence, into chunks of 64 tokens (the last one may be
// ragged).  cu_chunks[i] = sum_{j<i} ceil(len_j / 64) numbers the chunks globally; the intra-chunk
// kernels run one work item per (global chunk, head) of a window [win_lo, win_hi), the inter-chunk
// kernels one CTA per (sequence, head, dv-slice) walking that sequence's chunks in the window.
#pragma once

#include "kda_device.cuh"

namespace kda {

struct ChunkLoc {
    int seq;        // sequence index
    int chunk;      // chunk index inside the sequence
    long long tok0; // first token (global row) of the chunk
    int n;          // valid tokens in the chunk (1..64)
};

// Largest i in [0, n_seqs) with cu_chunks[i] <= gc (gc < cu_chunks[n_seqs]).
__device__ __forceinline__ int find_seq(const int32_t* __restrict__ cu_chunks, int n_seqs, long long gc) {
    int lo = 0, hi = n_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu_chunks[mid] <= gc) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ bool locate_chunk(const int32_t* __restrict__ cu_chunks,
                                             const int32_t* __restrict__ cu_seqlens, int n_seqs, long long gc,
                                             ChunkLoc& loc) {
    if (n_seqs <= 0 || gc >= cu_chunks[n_seqs]) return false;
    const int i = find_seq(cu_chunks, n_seqs, gc);
    loc.seq = i;
    loc.chunk = static_cast<int>(gc - cu_chunks[i]);
    const long long start = cu_seqlens[i];
    const long long len = static_cast<long long>(cu_seqlens[i + 1]) - start;
    loc.tok0 = start + static_cast<long long>(loc.chunk) * kChunk;
    const long long rem = len - static_cast<long long>(loc.chunk) * kChunk;
    loc.n = static_cast<int>(rem < kChunk ? rem : kChunk);
    return loc.n > 0;
}

}  // namespace kda
