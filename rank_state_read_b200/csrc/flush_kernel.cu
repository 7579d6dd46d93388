// Flush: the write-full step (one launch every W decode steps).
//
// Paper abstract (SketchSSM): the method "preserves full-state updates", and "at
// each state update ... reads the full state once to precompute outputs for these
// basis vectors, storing them in a compact sketch".  For every (batch row, head):
//   1. apply the n buffered tokens in order, S <- M_i S + beta_i k_i v_i^T
//      (Mamba-2 in closed form: S <- P S + sum_i w_i k_i v_i^T with
//       P = prod_i a_i, w_i = prod_{j>i} a_j);
//   2. write S back (skipped when n = 0);
//   3. for a sketch head, Y[off + m] = Omega_g[m] S for m < rank, from the S still
//      held in registers, so S crosses HBM once each way.
//
// One CTA per (b, h) with 2V threads.  Thread (ks, c4) holds the float4 column
// chunk c4 of the 16 state rows k = 8 j + ks (j < 16); a warp covers 4 column
// chunks x 8 row slices, so the reductions over k (the delta-rule erase term
// k^T S and the projection Omega S) are 3 xor-shuffle steps inside the warp.
// The buffered tokens and the head's basis rows are staged in shared memory.
#include "device_util.cuh"
#include "internal.cuh"

namespace sk {
namespace {

constexpr int ROWS_PER_THREAD = KDIM / 8;  // 16

template <int KIND>
__global__ void __launch_bounds__(2 * MAX_V)
flush_kernel(const FlushArgs A)
{
    extern __shared__ __align__(16) float fsm[];
    const int H = A.H, V = A.V, W = A.W, n = A.n;
    const long long bh = blockIdx.x;
    const int b = (int)(bh / H), h = (int)(bh - (long long)b * H);
    const int qk = h / A.hpq, g = h / A.Hg;
    const int r = __ldg(A.rank + h);
    const bool sketch = r > 0;
    if (n == 0 && !sketch) return;  // nothing to apply, nothing to project

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int V4 = V >> 2;
    float *kt = fsm;                       // [W][K] keys (Mamba-2: scaled by w_i)
    float *vt = kt + W * KDIM;             // [W][V] values
    float *sc = vt + W * V;                // [2W, padded to 4]: a_i (Mamba-2: w_i; sc[W] = P), beta_i
    float *av = sc + ((2 * W + 3) & ~3);   // KDA: [W][K] per-channel decays
    float *om = av + (KIND == SKETCHSSM_KDA ? W * KDIM : 0);  // [cap][K] basis rows

    if (tid < n) {
        sc[tid] = (KIND == SKETCHSSM_KDA) ? 0.f : __ldg(A.abuf + bh * W + tid);
        if (KIND != SKETCHSSM_MAMBA2) sc[W + tid] = __ldg(A.bbuf + bh * W + tid);
    }
    __syncthreads();
    if (KIND == SKETCHSSM_MAMBA2 && tid == 0) {
        float p = 1.f;
        for (int i = n - 1; i >= 0; --i) {
            const float ai = sc[i];
            sc[i] = p;  // w_i = prod_{j>i} a_j
            p *= ai;
        }
        sc[W] = p;      // P = prod_i a_i
    }
    __syncthreads();

    const long long krow = ((long long)b * A.Hqk + qk) * W;
    for (int x = tid; x < n * (KDIM / 4); x += blockDim.x) {
        const int i = x / (KDIM / 4), c = x - i * (KDIM / 4);
        float4 kv = ldg4(A.kbuf + (krow + i) * KDIM + c * 4);
        if (KIND == SKETCHSSM_MAMBA2) {
            const float w = sc[i];
            kv.x *= w; kv.y *= w; kv.z *= w; kv.w *= w;
        }
        st4(kt + i * KDIM + c * 4, kv);
        if (KIND == SKETCHSSM_KDA) st4(av + i * KDIM + c * 4, ldg4(A.abuf + (bh * W + i) * KDIM + c * 4));
    }
    for (int x = tid; x < n * V4; x += blockDim.x) {
        const int i = x / V4, c = x - i * V4;
        st4(vt + i * V + c * 4, ldg4(A.vbuf + (bh * W + i) * V + c * 4));
    }
    if (sketch) {
        const float *og = A.omega + (long long)g * A.Rb * KDIM;
        for (int x = tid; x < r * (KDIM / 4); x += blockDim.x) st4(om + x * 4, ldg4(og + x * 4));
    }
    __syncthreads();

    const int ks = lane & 7;
    const int c4 = warp * 4 + (lane >> 3);
    float *Sg = A.S + bh * KDIM * V + c4 * 4;
    float4 s[ROWS_PER_THREAD];
#pragma unroll
    for (int j = 0; j < ROWS_PER_THREAD; ++j) s[j] = ldg4(Sg + (long long)(j * 8 + ks) * V);

    if (KIND == SKETCHSSM_MAMBA2) {
        if (n > 0) {
            const float P = sc[W];
#pragma unroll
            for (int j = 0; j < ROWS_PER_THREAD; ++j) {
                s[j].x *= P; s[j].y *= P; s[j].z *= P; s[j].w *= P;
            }
            for (int i = 0; i < n; ++i) {
                const float4 vv = lds4(vt + i * V + c4 * 4);
                const float *ki = kt + i * KDIM + ks;
#pragma unroll
                for (int j = 0; j < ROWS_PER_THREAD; ++j) fma4(s[j], ki[j * 8], vv);
            }
        }
    } else {
        for (int i = 0; i < n; ++i) {
            const float *ki = kt + i * KDIM + ks;
            float4 d = zero4();
#pragma unroll
            for (int j = 0; j < ROWS_PER_THREAD; ++j) fma4(d, ki[j * 8], s[j]);
            d = sum8_xor(d);  // d = S^T k_i for this column chunk
            const float4 vv = lds4(vt + i * V + c4 * 4);
            const float bi = sc[W + i];
            if (KIND == SKETCHSSM_GDN) {
                // a (S - beta k d) + beta k v = a S + k * beta (v - a d)
                const float ai = sc[i];
                const float4 u = make_float4(bi * fmaf(-ai, d.x, vv.x), bi * fmaf(-ai, d.y, vv.y),
                                             bi * fmaf(-ai, d.z, vv.z), bi * fmaf(-ai, d.w, vv.w));
#pragma unroll
                for (int j = 0; j < ROWS_PER_THREAD; ++j) {
                    const float kk = ki[j * 8];
                    s[j].x = fmaf(ai, s[j].x, kk * u.x);
                    s[j].y = fmaf(ai, s[j].y, kk * u.y);
                    s[j].z = fmaf(ai, s[j].z, kk * u.z);
                    s[j].w = fmaf(ai, s[j].w, kk * u.w);
                }
            } else {
                // a_k (S - beta k_k d) + beta k_k v = a_k S + beta k_k (v - a_k d)
                const float *ai = av + i * KDIM + ks;
#pragma unroll
                for (int j = 0; j < ROWS_PER_THREAD; ++j) {
                    const float ak = ai[j * 8];
                    const float kb = bi * ki[j * 8];
                    s[j].x = fmaf(ak, s[j].x, kb * fmaf(-ak, d.x, vv.x));
                    s[j].y = fmaf(ak, s[j].y, kb * fmaf(-ak, d.y, vv.y));
                    s[j].z = fmaf(ak, s[j].z, kb * fmaf(-ak, d.z, vv.z));
                    s[j].w = fmaf(ak, s[j].w, kb * fmaf(-ak, d.w, vv.w));
                }
            }
        }
    }
    if (n > 0) {
#pragma unroll
        for (int j = 0; j < ROWS_PER_THREAD; ++j) st4(Sg + (long long)(j * 8 + ks) * V, s[j]);
    }
    if (sketch) {
        float *Yh = A.Y + ((long long)b * A.rtot + __ldg(A.off + h)) * V + c4 * 4;
        for (int m = 0; m < r; ++m) {
            const float *o = om + m * KDIM + ks;
            float4 p = zero4();
#pragma unroll
            for (int j = 0; j < ROWS_PER_THREAD; ++j) fma4(p, o[j * 8], s[j]);
            p = sum8_xor(p);
            if (ks == (m & 7)) st4(Yh + (long long)m * V, p);
        }
    }
}

template <int KIND>
cudaError_t launch_kind(const FlushArgs &a, cudaStream_t stream)
{
    const size_t smem = flush_smem_bytes(KIND, a.V, a.W, a.cap);
    cudaError_t e = cudaFuncSetAttribute(flush_kernel<KIND>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)a.B * a.H;
    flush_kernel<KIND><<<(unsigned)blocks, flush_threads(a.V), smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

int flush_threads(int V) { return 2 * V; }

size_t flush_smem_bytes(int kind, int V, int W, int cap)
{
    size_t f = (size_t)W * KDIM + (size_t)W * V + (size_t)((2 * W + 3) & ~3) + (size_t)cap * KDIM;
    if (kind == SKETCHSSM_KDA) f += (size_t)W * KDIM;
    return f * sizeof(float);
}

cudaError_t launch_flush(const FlushArgs &a, cudaStream_t stream)
{
    if (a.B == 0) return cudaSuccess;
    switch (a.kind) {
    case SKETCHSSM_MAMBA2: return launch_kind<SKETCHSSM_MAMBA2>(a, stream);
    case SKETCHSSM_GDN: return launch_kind<SKETCHSSM_GDN>(a, stream);
    default: return launch_kind<SKETCHSSM_KDA>(a, stream);
    }
}

}  // namespace sk
