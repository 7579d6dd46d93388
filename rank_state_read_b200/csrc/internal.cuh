// Internal declarations shared by the host API and the kernels of libsketchssm.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "sketchssm.h"

namespace sk {

constexpr int KDIM = 128;        // key dim the kernels are built for (Nemotron Nano card)
constexpr int MAX_HG = 32;       // heads per basis group
constexpr int MAX_W = 32;        // buffer window
constexpr int MAX_V = 256;       // value dim

// bits of the plan's device status word
constexpr int SK_STATUS_DECODE_TIMEOUT = 1;
constexpr int SK_STATUS_FLUSH_TIMEOUT = 2;
constexpr int SK_STATUS_STEP_TIMEOUT = 4;
constexpr int SK_STATUS_BAD_ROW = 8;  // a per-row position or token count out of range
constexpr int SK_STATUS_PREFILL_TIMEOUT = 16;

// default bound of a kernel's wait on its own bulk copies (clock cycles, ~1 s)
constexpr long long DEFAULT_WAIT_CYCLES = 2000000000LL;

// Arguments of one decode step (sketch or dense-read): coefficient + combine launches.
struct DecodeArgs {
    int kind, B, H, Hqk, V, W, G, Rb, cap, pos;
    int Hg;              // heads per group
    int hpq;             // heads per q/k head
    int64_t rtot;        // sketch rows per batch row
    const int *rank, *off;
    const int *coff;     // coefficient block of each head within a batch row (sketch layout)
    int coef_row;        // coefficient floats per batch row (of the layout in use)
    int coef_dense_block;// per-head block of the dense-read layout (head h at h * block)
    float *scratch;      // Mamba-2: products, B x Hqk x dots_row; GDN/KDA: coefficients, B x coef_row
    const int *work;     // combine items of this step (already offset to its n)
    const int *rec;      // their records, 8 ints each (layout kernel)
    const int *qk_rneed; // largest sketch rank per q/k head
    int n_items;         // combine items per batch row
    int dense_all;       // 1: every head reads its state (dense-read baseline)
    int threads;         // combine CTA size
    int stage_rows;      // rows of the combine stage
    int cm_rows;         // batch rows per Mamba-2 product CTA
    int dots_row;        // Mamba-2 products per (batch row, q/k head): W keys, then cap basis rows
    int maxnh;           // heads per combine item at most
    int coef_cap;        // floats of the combine coefficient stage
    const int *row_pos;  // per-row buffer positions [B] (device), or null: every row at pos
    const int *counts;   // layout counts: items of the work list for n at counts[2 + n]
    long long wait_limit;
    int *status;
    const float *q, *k, *v, *a, *beta;
    float *kbuf, *vbuf, *abuf, *bbuf;
    const float *Y, *omega, *S;
    float *y;
};

// Arguments of one flush launch.
struct FlushArgs {
    int kind, B, H, Hqk, V, W, G, Rb, cap, n;
    int Hg, hpq;
    int VS;    // column slab of one work item
    const int *row_n;  // per-row token counts [B] (device), or null: every row applies n
    int rcap;  // the largest sketch rank of the plan (0 if none): basis rows staged per CTA
    const int *rmax;          // [G] largest sketch rank per group
    int *status;              // plan status word (timeouts)
    long long wait_limit;     // clock cycles of a bounded wait
    int64_t rtot;
    const int *rank, *off;
    float *S;
    const float *omega, *kbuf, *vbuf, *abuf, *bbuf;
    float *Y;
};

// Geometry of the combine launch for a layer shape: heads per item, CTA size, rows of
// one shared-memory stage (the packing budget of a sketch item), coefficient stage.
struct DecodeGeometry {
    int maxnh, threads, stage_rows, coef_cap;
};
bool decode_geometry(int kind, int V, int W, int cap, int Hg, DecodeGeometry *gm);
int coef_block(int rows, int W);  // floats of one head's coefficient block
int coef_rows(int cap, int W, int B, int Hqk, int sms);  // batch rows per Mamba-2 products CTA
int dots_row(int W, int cap);
size_t decode_smem_bytes(const DecodeArgs &a);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);


// Arguments of one standard per-step decode launch.
struct StepArgs {
    int kind, B, H, Hqk, V, hpq;
    int VS;  // column slab of one CTA
    long long wait_limit;
    int *status;
    const float *q, *k, *v, *a, *beta;
    float *S, *y;
};
int step_slab(int V);
cudaError_t launch_step(const StepArgs &a, cudaStream_t stream);

// Prefill: a prompt of T tokens (token-major k [B][T][Hqk][K], v [B][T][H][V],
// a [B][T][H] or KDA [B][T][H][K], beta [B][T][H]) applied to S in place; the column
// slab VS follows step_slab.
struct PrefillArgs {
    int kind, B, H, Hqk, V, hpq, T;
    int VS;
    const float *k, *v, *a, *beta;
    float *S;
    int *status;           // plan status word (timeouts of the tensor-core waits)
    long long wait_limit;  // clock cycles of a bounded wait
};
cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t stream);
// Mamba-2 prompts of at most 64 tokens with V a multiple of 16 up to 128: the tcgen05 kernel
bool prefill_tcgen05_fits(const PrefillArgs &a);
cudaError_t launch_prefill_tcgen05(const PrefillArgs &a, cudaStream_t stream);

int flush_slab(int V);
size_t flush_smem_bytes(int kind, int V, int W, int rcap);
cudaError_t launch_flush(const FlushArgs &a, cudaStream_t stream);

// Layout kernel: off[H+1], rmax[G], coff[H], per-n work lists work[(n-1)(H+G) ...];
// counts = {dense heads, invalid-rank flag, coefficient floats per row, items for
// n = 1 .. W}.
cudaError_t launch_layout(const int *rank, int H, int G, int Hqk, int W, int cap, int row_budget, int max_heads,
                          int *off, int *rmax, int *coff, int *work, int *rec, int *qk_rneed, int *counts,
                          cudaStream_t stream);

}  // namespace sk

struct sketchssm_plan {
    sketchssm_desc d;
    int Hg, hpq;
    int64_t rtot;
    int n_dense;
    sk::DecodeGeometry geo;
    int device;
    int sms;  // SMs of the plan's device
    long long wait_limit;
    int coef_row;
    int *d_rank, *d_off, *d_rmax, *d_coff, *d_work, *d_rec, *d_qk_rneed, *d_counts, *d_status;
    float *d_scratch;
    size_t scratch_floats;
    std::vector<int32_t> h_rank, h_off, h_rmax, h_work, h_items;
};
