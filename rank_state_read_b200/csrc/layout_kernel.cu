// Rank/group-aware launch layout (one CTA, runs once per plan).
//
// From the per-head rank table (a rank or a dense fallback per head, sketchssm
// PyPI page, calibration stage "allocate") and the contiguous basis groups (stage
// "basis": one shared basis per head group), compute
//   off[h]   exclusive prefix sum of the sketch ranks (dense heads own no sketch row),
//   off[H]   Rtot, the sketch rows of one batch row,
//   rmax[g]  the largest sketch rank of group g (0 if none),
//   coff[h] the head's coefficient block within a batch row: sketch heads first, in
//            head order, round4(r_h + W) floats each, then the dense heads,
//            round4(K + W) floats each (so the blocks of consecutive sketch heads are
//            one contiguous range),
//   work     for every n = 1..W (tokens replayed by a decode step), the combine items
//            of one batch row: first every dense head in head order (entry -h-1),
//            then per group the sketch heads packed greedily, in head order, into
//            items of at most `max_heads` heads whose rows (r_h + n per head) stay
//            within `row_budget` (entry first_head * 64 + span,
//            span = last - first + 1),
//   rec      per work entry a record of 8 ints {entry, span, member mask, rows R,
//            first sketch row off[h_first], coefficient offset coff[h_first],
//            coefficient floats of the item, h_first}, so that a combine CTA can issue
//            its copies after a single table load,
//   qk_rneed the largest sketch rank among the heads of each q/k head (0 if none),
//   counts   {dense heads, invalid-rank flag, coefficient floats per batch row,
//            items for n = 1, ..., items for n = W}.
// The row budget is one shared-memory stage of the combine kernel, so every item is
// staged at once; items are balanced by bytes, not by heads.
// Integer only; the host compares it bit for bit with its definition.
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
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        warp_sums[lane] = wi - w;  // exclusive prefix of the warp sums
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    const int res = warp_sums[warp] + incl - x;
    __syncthreads();  // warp_sums is reused by the next call
    return res;
}

__device__ __forceinline__ int round4(int x) { return (x + 3) & ~3; }

// Greedy packing of group g's sketch heads for n replayed tokens.  Writes the items'
// entries to out (if not null) and returns their count.
__device__ int pack_group(const int *rank, int g, int Hg, int n, int row_budget, int max_heads, int *out)
{
    int count = 0, first = -1, last = -1, heads = 0, rows = 0;
    for (int h = g * Hg; h < (g + 1) * Hg; ++h) {
        const int r = rank[h];
        if (r <= 0) continue;
        const int need = r + n;
        if (heads > 0 && (rows + need > row_budget || heads == max_heads)) {
            if (out) out[count] = first * 64 + (last - first + 1);
            ++count;
            heads = 0;
            rows = 0;
        }
        if (heads == 0) first = h;
        rows += need;
        last = h;
        ++heads;
    }
    if (heads > 0) {
        if (out) out[count] = first * 64 + (last - first + 1);
        ++count;
    }
    return count;
}

__global__ void __launch_bounds__(LAYOUT_THREADS)
layout_kernel(const int *__restrict__ rank, int H, int G, int Hqk, int W, int cap, int row_budget,
              int max_heads, int *__restrict__ off, int *__restrict__ rmax, int *__restrict__ coff,
              int *__restrict__ work, int *__restrict__ rec, int *__restrict__ qk_rneed,
              int *__restrict__ counts)
{
    __shared__ int warp_sums[32];
    __shared__ int total;
    __shared__ int carry_rows, carry_dense, carry_coef, bad;
    const int Hg = H / G;
    const int stride = H + G;  // entries per n
    if (threadIdx.x == 0) {
        carry_rows = 0;
        carry_dense = 0;
        carry_coef = 0;
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
        const int ex_coef = block_exclusive_scan(rows > 0 ? round4(rows + W) : 0, warp_sums, &total);
        const int tot_coef = total;
        if (h < H) {
            off[h] = carry_rows + ex_rows;
            coff[h] = rows > 0 ? carry_coef + ex_coef : -1 - (carry_dense + ex_dense);
            if (isd)
                for (int n = 1; n <= W; ++n) work[(n - 1) * stride + carry_dense + ex_dense] = -h - 1;
            if (rows > 0) atomicMax(&rmax[h / Hg], r);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            carry_rows += tot_rows;
            carry_dense += tot_dense;
            carry_coef += tot_coef;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) off[H] = carry_rows;
    __syncthreads();
    const int n_dense = carry_dense;
    const int sketch_coef = carry_coef;
    for (int h = threadIdx.x; h < H; h += blockDim.x)  // dense blocks follow the sketch blocks
        if (coff[h] < 0) coff[h] = sketch_coef + (-1 - coff[h]) * round4(KDIM + W);

    for (int n = 1; n <= W; ++n) {
        int *list = work + (n - 1) * stride + n_dense;
        int carry = 0;
        for (int base = 0; base < G; base += blockDim.x) {
            const int g = base + threadIdx.x;
            const int c = (g < G) ? pack_group(rank, g, Hg, n, row_budget, max_heads, nullptr) : 0;
            const int ex = block_exclusive_scan(c, warp_sums, &total);
            const int tot = total;
            if (g < G && c > 0) pack_group(rank, g, Hg, n, row_budget, max_heads, list + carry + ex);
            carry += tot;
        }
        if (threadIdx.x == 0) counts[2 + n] = n_dense + carry;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        counts[0] = n_dense;
        counts[1] = bad;
        counts[2] = sketch_coef + n_dense * round4(KDIM + W);
    }
    // records of the work entries
    for (int n = 1; n <= W; ++n) {
        const int items = counts[2 + n];
        for (int i = threadIdx.x; i < items; i += blockDim.x) {
            const int e = work[(n - 1) * stride + i];
            int *o = rec + ((size_t)(n - 1) * stride + i) * 8;
            if (e < 0) {
                const int h = -e - 1;
                o[0] = e; o[1] = 1; o[2] = 1; o[3] = KDIM; o[4] = 0;
                o[5] = coff[h]; o[6] = round4(KDIM + W); o[7] = h;
            } else {
                const int hf = e >> 6, span = e & 63, last = hf + span - 1;
                unsigned mask = 0;
                for (int l = 0; l < span; ++l)
                    if (rank[hf + l] > 0) mask |= 1u << l;
                o[0] = e; o[1] = span; o[2] = (int)mask; o[3] = off[hf + span] - off[hf]; o[4] = off[hf];
                o[5] = coff[hf]; o[6] = coff[last] + round4(rank[last] + W) - coff[hf]; o[7] = hf;
            }
        }
    }
    // the largest sketch rank of each q/k head's heads
    const int hpq = H / Hqk;
    for (int q = threadIdx.x; q < Hqk; q += blockDim.x) {
        int m = 0;
        for (int l = 0; l < hpq; ++l) m = max(m, rank[q * hpq + l]);
        qk_rneed[q] = m;
    }
}

}  // namespace

cudaError_t launch_layout(const int *rank, int H, int G, int Hqk, int W, int cap, int row_budget, int max_heads,
                          int *off, int *rmax, int *coff, int *work, int *rec, int *qk_rneed, int *counts,
                          cudaStream_t stream)
{
    cudaError_t e = cudaMemsetAsync(counts, 0, (3 + W) * sizeof(int), stream);
    if (e != cudaSuccess) return e;
    layout_kernel<<<1, LAYOUT_THREADS, 0, stream>>>(rank, H, G, Hqk, W, cap, row_budget, max_heads, off, rmax,
                                                    coff, work, rec, qk_rneed, counts);
    return cudaGetLastError();
}

}  // namespace sk
