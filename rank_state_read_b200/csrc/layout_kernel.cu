// Rank/group-aware launch layout (one CTA, runs once per plan).
//
// From the per-head rank table (a rank or a dense fallback per head, sketchssm
// PyPI page, calibration stage "allocate") and the contiguous basis groups (stage
// "basis": one shared basis per head group), compute
//   off[h]  exclusive prefix sum of the sketch ranks (dense heads own no sketch row),
//   off[H]  Rtot, the sketch rows of one batch row,
//   rmax[g] the largest sketch rank of group g (0 if none),
//   work[]  the CTA items of one batch row of the decode launch: every dense head in
//           head order (entry -h-1), then every group that holds a sketch head, in
//           group order (entry g),
//   counts  {items, dense heads, invalid-rank flag, largest group sketch rows}.
// Integer only; the host compares it bit for bit with the oracle's layout.
#include "internal.cuh"

namespace sk {
namespace {

constexpr int LAYOUT_THREADS = 1024;

// Exclusive block scan of one int per thread; returns the exclusive prefix and
// writes the block total to *total.  All threads of the block must call it.
__device__ int block_exclusive_scan(int x, int *warp_sums, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        warp_sums[lane] = wi - w;  // exclusive prefix of the warp sums
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    int res = warp_sums[warp] + incl - x;
    __syncthreads();  // warp_sums is reused by the next call
    return res;
}

__global__ void __launch_bounds__(LAYOUT_THREADS)
layout_kernel(const int *__restrict__ rank, int H, int G, int cap, int *__restrict__ off,
              int *__restrict__ rmax, int *__restrict__ work, int *__restrict__ counts)
{
    __shared__ int warp_sums[32];
    __shared__ int total;
    __shared__ int carry_rows, carry_dense, bad;
    const int Hg = H / G;
    if (threadIdx.x == 0) {
        carry_rows = 0;
        carry_dense = 0;
        bad = 0;
    }
    for (int g = threadIdx.x; g < G; g += blockDim.x) rmax[g] = 0;
    __syncthreads();

    for (int base = 0; base < H; base += blockDim.x) {
        const int h = base + threadIdx.x;
        const int r = (h < H) ? rank[h] : 0;
        if (h < H && !(r == SKETCHSSM_DENSE || (r >= 1 && r <= cap))) atomicOr(&bad, 1);
        const int rows = (h < H && r > 0) ? r : 0;
        const int isd = (h < H && r == SKETCHSSM_DENSE) ? 1 : 0;
        const int ex_rows = block_exclusive_scan(rows, warp_sums, &total);
        const int tot_rows = total;
        const int ex_dense = block_exclusive_scan(isd, warp_sums, &total);
        const int tot_dense = total;
        if (h < H) {
            off[h] = carry_rows + ex_rows;
            if (isd) work[carry_dense + ex_dense] = -h - 1;
            if (rows > 0) atomicMax(&rmax[h / Hg], r);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            carry_rows += tot_rows;
            carry_dense += tot_dense;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) off[H] = carry_rows;
    __syncthreads();

    // group items after the dense items, in group order
    int carry_groups = 0;
    for (int base = 0; base < G; base += blockDim.x) {
        const int g = base + threadIdx.x;
        const int has = (g < G && rmax[g] > 0) ? 1 : 0;
        const int ex = block_exclusive_scan(has, warp_sums, &total);
        const int tot = total;
        if (has) {
            work[carry_dense + carry_groups + ex] = g;
            const int rows = off[(g + 1) * Hg] - off[g * Hg];
            atomicMax(&counts[3], rows);
        }
        carry_groups += tot;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        counts[0] = carry_dense + carry_groups;
        counts[1] = carry_dense;
        counts[2] = bad;
    }
}

}  // namespace

cudaError_t launch_layout(const int *rank, int H, int G, int cap, int *off, int *rmax, int *work,
                          int *counts, cudaStream_t stream)
{
    cudaError_t e = cudaMemsetAsync(counts, 0, 4 * sizeof(int), stream);
    if (e != cudaSuccess) return e;
    layout_kernel<<<1, LAYOUT_THREADS, 0, stream>>>(rank, H, G, cap, off, rmax, work, counts);
    return cudaGetLastError();
}

}  // namespace sk
