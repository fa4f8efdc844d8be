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

// dstart[b*T + t] = start of the run of equal ids containing t: an inclusive max-scan of
// (t if t starts a run, else -1) along the row.  One block per batch row, chunks of blockDim.x
// positions, the running maximum carried between chunks.  blockDim.x is a multiple of 32, <= 1024.
__global__ void doc_start_kernel(const int* __restrict__ doc, int* __restrict__ dstart, int T) {
    __shared__ int warp_max[32];
    __shared__ int carry;
    const int b = blockIdx.x;
    const int* d = doc + (long long)b * T;
    int* o = dstart + (long long)b * T;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < T; base += blockDim.x) {
        const int t = base + threadIdx.x;
        int v = -1;
        if (t < T) v = (t == 0 || d[t] != d[t - 1]) ? t : -1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v = max(v, u);
        }
        if (lane == 31) warp_max[warp] = v;
        __syncthreads();
        if (warp == 0) {
            int w = lane < nwarps ? warp_max[lane] : -1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, w, off);
                if (lane >= off) w = max(w, u);
            }
            warp_max[lane] = w;
        }
        __syncthreads();
        v = max(v, max(warp > 0 ? warp_max[warp - 1] : -1, carry));
        if (t < T) o[t] = v;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = v;
        __syncthreads();
    }
}

}  // namespace swa
