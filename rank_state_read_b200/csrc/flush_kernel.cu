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
// One CTA per (b, h, column slab of VS <= 128 columns); columns of S evolve
// independently, so a slab is self-contained.  2 VS threads: thread (ks, c4) holds
// the float4 column chunk c4 of the 16 consecutive state rows 16 ks .. 16 ks + 15,
// and a warp covers 4 column chunks x 8 row slices, so every reduction over k (the
// delta-rule erase term k^T S and the projection Omega S) is 3 xor-shuffle steps
// inside the warp.  The state loads are issued first, straight into registers, and
// fly while the CTA stages the buffered tokens in shared memory; keys and KDA decays
// are staged with 4 floats of padding per 16 so that the float4 reads of the 8 row
// slices fall on disjoint banks.  The basis rows are read through L1.
#include "device_util.cuh"
#include "internal.cuh"

namespace sk {
namespace {

constexpr int RPT = KDIM / 8;          // state rows per thread (16)
constexpr int KPAD = KDIM + KDIM / 4;  // padded key row: 4 pad floats per 16

__device__ __forceinline__ int kpad(int k) { return k + (k >> 4) * 4; }

__host__ __device__ inline size_t flush_smem_floats(int kind, int VS, int W)
{
    return (size_t)W * KPAD + (size_t)W * VS + 2 * (size_t)W + (kind == SKETCHSSM_KDA ? (size_t)W * KPAD : 0);
}

template <int KIND, int MAXT, int MINB>
__global__ void __launch_bounds__(MAXT, MINB)
flush_kernel(const FlushArgs A)
{
    extern __shared__ __align__(16) float fsm[];
    const int H = A.H, V = A.V, W = A.W, n = A.n, VS = A.VS;
    const int nslab = V / VS;
    const long long item = blockIdx.x;
    const long long bh = item / nslab;
    const int slab = (int)(item - bh * nslab);
    const int b = (int)(bh / H), h = (int)(bh - (long long)b * H);
    const int r = __ldg(A.rank + h);
    if (n == 0 && r <= 0) return;  // nothing to apply, nothing to project

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, T = blockDim.x;
    const int ks = lane & 7;
    const int c4 = warp * 4 + (lane >> 3);

    // 1. the state slab, straight into registers
    float *Sg = A.S + (bh * KDIM + ks * RPT) * V + slab * VS + c4 * 4;
    float4 s[RPT];
#pragma unroll
    for (int j = 0; j < RPT; ++j) s[j] = ldg4(Sg + (long long)j * V);

    // 2. buffered tokens into shared memory
    float *kt = fsm;                 // [W][KPAD] keys
    float *vt = kt + W * KPAD;       // [W][VS]   values of the slab
    float *sc = vt + W * VS;         // [2W]      a_i (or alpha_i), beta_i
    float *av = sc + 2 * W;          // [W][KPAD] KDA decays
    if (n > 0) {
        const int qk = h / A.hpq;
        const float *kg = A.kbuf + ((long long)b * A.Hqk + qk) * W * KDIM;
        for (int x = tid; x < n * (KDIM / 4); x += T) {
            const int i = x / (KDIM / 4), c = x - i * (KDIM / 4);
            st4(kt + i * KPAD + kpad(c * 4), ldg4(kg + (long long)i * KDIM + c * 4));
            if (KIND == SKETCHSSM_KDA)
                st4(av + i * KPAD + kpad(c * 4), ldg4(A.abuf + (bh * W + i) * KDIM + c * 4));
        }
        const int VS4 = VS / 4;
        for (int x = tid; x < n * VS4; x += T) {
            const int i = x / VS4, c = x - i * VS4;
            st4(vt + i * VS + c * 4, ldg4(A.vbuf + (bh * W + i) * V + slab * VS + c * 4));
        }
        if (tid < n) {
            if (KIND != SKETCHSSM_KDA) sc[tid] = __ldg(A.abuf + bh * W + tid);
            if (KIND != SKETCHSSM_MAMBA2) sc[W + tid] = __ldg(A.bbuf + bh * W + tid);
        }
    }
    __syncthreads();

    // 3. the update
    const float *ktr = kt + ks * 20;  // = kpad(16 ks)
    if (KIND == SKETCHSSM_MAMBA2) {
        if (n > 0) {
            float P = 1.f;
            for (int i = 0; i < n; ++i) P *= sc[i];
#pragma unroll
            for (int j = 0; j < RPT; ++j) {
                s[j].x *= P; s[j].y *= P; s[j].z *= P; s[j].w *= P;
            }
            float w = 1.f;  // w_i = prod_{j>i} a_j, newest token first
            for (int i = n - 1; i >= 0; --i) {
                float4 vv = lds4(vt + i * VS + c4 * 4);
                vv.x *= w; vv.y *= w; vv.z *= w; vv.w *= w;
                const float *ki = ktr + i * KPAD;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 kk = lds4(ki + q * 4);
                    fma4(s[4 * q + 0], kk.x, vv);
                    fma4(s[4 * q + 1], kk.y, vv);
                    fma4(s[4 * q + 2], kk.z, vv);
                    fma4(s[4 * q + 3], kk.w, vv);
                }
                w *= sc[i];
            }
        }
    } else {
        const float *avr = av + ks * 20;
        for (int i = 0; i < n; ++i) {
            const float *ki = ktr + i * KPAD;
            float4 d = zero4();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 kk = lds4(ki + q * 4);
                fma4(d, kk.x, s[4 * q + 0]);
                fma4(d, kk.y, s[4 * q + 1]);
                fma4(d, kk.z, s[4 * q + 2]);
                fma4(d, kk.w, s[4 * q + 3]);
            }
            d = sum8_xor(d);  // d = S^T k_i for this column chunk
            const float4 vv = lds4(vt + i * VS + c4 * 4);
            const float bi = sc[W + i];
            if (KIND == SKETCHSSM_GDN) {
                // a (S - beta k d) + beta k v = a S + k * beta (v - a d)
                const float ai = sc[i];
                const float4 u = make_float4(bi * fmaf(-ai, d.x, vv.x), bi * fmaf(-ai, d.y, vv.y),
                                             bi * fmaf(-ai, d.z, vv.z), bi * fmaf(-ai, d.w, vv.w));
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 kk = lds4(ki + q * 4);
                    const float kq[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float4 &t = s[4 * q + e];
                        t.x = fmaf(ai, t.x, kq[e] * u.x);
                        t.y = fmaf(ai, t.y, kq[e] * u.y);
                        t.z = fmaf(ai, t.z, kq[e] * u.z);
                        t.w = fmaf(ai, t.w, kq[e] * u.w);
                    }
                }
            } else {
                // a_k (S - beta k_k d) + beta k_k v = a_k S + beta k_k (v - a_k d)
                const float *ai = avr + i * KPAD;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 kk = lds4(ki + q * 4);
                    const float4 a4 = lds4(ai + q * 4);
                    const float kq[4] = {kk.x, kk.y, kk.z, kk.w};
                    const float aq[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float4 &t = s[4 * q + e];
                        const float ak = aq[e], kb = bi * kq[e];
                        t.x = fmaf(ak, t.x, kb * fmaf(-ak, d.x, vv.x));
                        t.y = fmaf(ak, t.y, kb * fmaf(-ak, d.y, vv.y));
                        t.z = fmaf(ak, t.z, kb * fmaf(-ak, d.z, vv.z));
                        t.w = fmaf(ak, t.w, kb * fmaf(-ak, d.w, vv.w));
                    }
                }
            }
        }
    }
    if (n > 0) {
#pragma unroll
        for (int j = 0; j < RPT; ++j) st4(Sg + (long long)j * V, s[j]);
    }

    // 4. the sketch rows of this slab, from registers
    if (r > 0) {
        float *Yh = A.Y + ((long long)b * A.rtot + __ldg(A.off + h)) * V + slab * VS + c4 * 4;
        const float *og = A.omega + ((long long)(h / A.Hg) * A.Rb) * KDIM + ks * RPT;
        for (int m = 0; m < r; ++m) {
            const float *o = og + (long long)m * KDIM;
            float4 p = zero4();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 om = ldg4(o + q * 4);
                fma4(p, om.x, s[4 * q + 0]);
                fma4(p, om.y, s[4 * q + 1]);
                fma4(p, om.z, s[4 * q + 2]);
                fma4(p, om.w, s[4 * q + 3]);
            }
            p = sum8_xor(p);
            if (ks == (m & 7)) st4(Yh + (long long)m * V, p);
        }
    }
}

template <int KIND, int MAXT, int MINB>
cudaError_t launch_cfg(const FlushArgs &a, cudaStream_t stream)
{
    const size_t smem = flush_smem_floats(KIND, a.VS, a.W) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(flush_kernel<KIND, MAXT, MINB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)a.B * a.H * (a.V / a.VS);
    flush_kernel<KIND, MAXT, MINB><<<(unsigned)blocks, 2 * a.VS, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int KIND>
cudaError_t launch_kind(const FlushArgs &a, cudaStream_t stream)
{
    // slabs of up to 80 columns run 160-thread CTAs, four per SM; wider slabs 256
    if (2 * a.VS <= 160) return launch_cfg<KIND, 160, 4>(a, stream);
    return launch_cfg<KIND, 256, 2>(a, stream);
}

}  // namespace

int flush_slab(int V)
{
    if (V <= 128) return V;
    for (int vs = 128; vs >= 16; vs -= 16)
        if (V % vs == 0) return vs;
    return 16;
}

size_t flush_smem_bytes(int kind, int V, int W)
{
    return flush_smem_floats(kind, flush_slab(V), W) * sizeof(float);
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
