// docmask.cuh -- document starts for the document-boundary mask.
//
// Reading taken (the pages name masking at document boundaries only as a change that was tried;
// intelliparadigm "GPT-2 for $73", section 7, the variable-length attention item): packed
// documents are the maximal runs of equal ids along a sequence, and key j is visible to query i
// iff 0 <= i - j < W and j lies in i's document, i.e. j >= start(i), the first position of the run
// that contains i.  RoPE positions stay the sequence positions.  For ids that never repeat across
// runs (packed documents numbered in order) this is "same id", the oracle's statement of the mask.
#pragma once

#include <cstdint>

namespace swa {

// Inclusive scan of one chunk of blockDim.x values (one per thread) under max (kMax) or min, the
// running value of earlier chunks folded in through `carry`.  blockDim.x is a multiple of 32 and at
// most 1024; every thread of the block calls it.
template <bool kMax>
__device__ __forceinline__ int block_scan_chunk(int v, int* warp_acc, int& carry) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    auto op = [](int a, int b) { return kMax ? max(a, b) : min(a, b); };
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v = op(v, u);
    }
    if (lane == 31) warp_acc[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? warp_acc[lane] : (kMax ? -1 : 0x7fffffff);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w = op(w, u);
        }
        warp_acc[lane] = w;
    }
    __syncthreads();
    v = op(v, op(warp > 0 ? warp_acc[warp - 1] : (kMax ? -1 : 0x7fffffff), carry));
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) warp_acc[0] = v;
    __syncthreads();
    carry = warp_acc[0];
    __syncthreads();
    return v;
}

// Per position t of each row: dstart = first position of the run of equal ids containing t (an
// inclusive max-scan of "t if a run starts at t, else -1"), and, when dend is not null, dend = last
// position of that run (a min-scan from the end of "t if a run ends at t, else +inf").  One block
// per batch row, chunks of blockDim.x positions.
__global__ void doc_start_kernel(const int* __restrict__ doc, int* __restrict__ dstart, int* __restrict__ dend,
                                 int T) {
    __shared__ int warp_acc[32];
    const int b = blockIdx.x;
    const int* d = doc + (long long)b * T;
    int carry = -1;
    for (int base = 0; base < T; base += blockDim.x) {
        const int t = base + threadIdx.x;
        const int v = (t < T && (t == 0 || d[t] != d[t - 1])) ? t : -1;
        const int r = block_scan_chunk<true>(v, warp_acc, carry);
        if (t < T) dstart[(long long)b * T + t] = r;
    }
    if (dend == nullptr) return;
    carry = 0x7fffffff;
    for (int base = 0; base < T; base += blockDim.x) {
        const int t = T - 1 - (base + threadIdx.x);          // walks the row from its end
        const int v = (t >= 0 && (t == T - 1 || d[t] != d[t + 1])) ? t : 0x7fffffff;
        const int r = block_scan_chunk<false>(v, warp_acc, carry);
        if (t >= 0) dend[(long long)b * T + t] = r;
    }
}

}  // namespace swa
