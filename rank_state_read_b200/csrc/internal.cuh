// Internal declarations shared by the host API and the kernels of libsketchssm.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "sketchssm.h"

namespace sk {

constexpr int KDIM = 128;        // key dim the kernels are built for (Nemotron Nano card)
constexpr int KDIM4 = KDIM / 4;  // float4 lanes of a key vector: one per warp lane
constexpr int MAX_HG = 32;       // heads per basis group
constexpr int MAX_W = 32;        // buffer window
constexpr int MAX_V = 256;       // value dim

// Arguments of one decode launch (sketch or dense-read).
struct DecodeArgs {
    int kind, B, H, Hqk, V, W, G, Rb, cap, pos;
    int Hg;        // heads per group
    int hpq;       // heads per q/k head
    int64_t rtot;  // sketch rows per batch row
    const int *rank, *off, *work;
    int n_work;    // items per batch row
    int dense_all; // 1: every head is a dense item (dense-read baseline)
    int ns;        // row slices of the weighted row sum
    int max_rows;  // capacity of the per-item row tables
    const float *q, *k, *v, *a, *beta;
    float *kbuf, *vbuf, *abuf, *bbuf;
    const float *Y, *omega, *S;
    float *y;
};

// Arguments of one flush launch.
struct FlushArgs {
    int kind, B, H, Hqk, V, W, G, Rb, cap, n;
    int Hg, hpq;
    int64_t rtot;
    const int *rank, *off;
    float *S;
    const float *omega, *kbuf, *vbuf, *abuf, *bbuf;
    float *Y;
};

// Dynamic shared memory of a decode CTA (bytes) and its thread count.
size_t decode_smem_bytes(const DecodeArgs &a);
int decode_threads(int V, int *ns_out);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

size_t flush_smem_bytes(int kind, int V, int W, int cap);
int flush_threads(int V);
cudaError_t launch_flush(const FlushArgs &a, cudaStream_t stream);

// Layout kernel: off[H+1], rmax[G], work[G+H]; counts = {n_work, n_dense, err, max_group_rows}.
cudaError_t launch_layout(const int *rank, int H, int G, int cap, int *off, int *rmax, int *work,
                          int *counts, cudaStream_t stream);

}  // namespace sk

struct sketchssm_plan {
    sketchssm_desc d;
    int Hg, hpq;
    int64_t rtot;
    int n_work, n_dense, max_group_rows;
    int device;
    int *d_rank, *d_off, *d_rmax, *d_work, *d_counts;
    std::vector<int32_t> h_rank, h_off, h_rmax, h_work;
};
