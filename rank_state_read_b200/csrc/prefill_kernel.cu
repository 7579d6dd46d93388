// Prefill handoff: the state after a prompt, the step before the decode path.  The
// paper's update is write-full (paper abstract: every state update reaches the full
// state); a prompt is taken in the same way, token after token: for every (batch row,
// head) apply t = 0 .. T-1 to S in place, S <- M_t S + beta_t k_t v_t^T (Mamba-2:
// M = a I, beta = 1; GDN: M = a (I - beta k k^T); KDA: M = diag(a) (I - beta k k^T)).
// The host then forms the sketch with the n = 0 flush.
//
// One CTA per (b, h, column slab of VS columns), 2 VS threads.  The slab stays in
// registers for the whole prompt (thread (ks, c4) holds the float4 column chunk c4 of
// the 16 state rows 4 ks + 32 q + e, q, e < 4), so S is read and written once however
// long the prompt; the delta rule's k^T S is 3 xor-shuffle steps inside the warp.  The
// prompt comes through shared memory in chunks of PF_CHUNK tokens, double buffered with
// cp.async: chunk c + 1 is in flight while the CTA applies chunk c.  No thread waits
// on another CTA or on a flag: the only waits are cp.async groups and CTA barriers.
#include "device_util.cuh"
#include "internal.cuh"
#include "ptx_util.cuh"

namespace sk {
namespace {

constexpr int PF_MAXT = 160;  // slabs of at most 80 columns
constexpr int PF_CHUNK = 16;  // tokens per shared-memory stage

struct PrefillCarve {
    size_t k, v, a, beta, total;  // each [2 stages][PF_CHUNK][...]
};

__host__ __device__ inline size_t pf_align(size_t x) { return (x + 127) & ~size_t(127); }

__host__ __device__ inline PrefillCarve prefill_carve(int kind, int VS)
{
    PrefillCarve c;
    size_t o = 0;
    c.k = o;
    o = pf_align(o + sizeof(float) * 2 * PF_CHUNK * KDIM);
    c.v = o;
    o = pf_align(o + sizeof(float) * 2 * PF_CHUNK * (size_t)VS);
    c.a = o;
    o = pf_align(o + sizeof(float) * 2 * PF_CHUNK * (kind == SKETCHSSM_KDA ? KDIM : 1));
    c.beta = o;
    o = pf_align(o + (kind == SKETCHSSM_MAMBA2 ? 0 : sizeof(float) * 2 * PF_CHUNK));
    c.total = o;
    return c;
}

// Issue the copies of tokens t0 .. t0 + n - 1 into one stage (no wait).
template <int KIND>
__device__ __forceinline__ void issue_chunk(const PrefillArgs &A, long long b, int h, int qk, int slab, int t0,
                                            int n, float *ks, float *vs, float *as, float *bs)
{
    const int tid = threadIdx.x, nthr = blockDim.x, VS = A.VS, vq = VS / 4;
    const long long tb = b * A.T + t0;  // token t0 of row b
    for (int x = tid; x < n * (KDIM / 4); x += nthr) {
        const int i = x >> 5, c = x & 31;
        cp_async16(ks + i * KDIM + c * 4, A.k + ((tb + i) * A.Hqk + qk) * KDIM + c * 4);
    }
    for (int x = tid; x < n * vq; x += nthr) {
        const int i = x / vq, c = x - i * vq;
        cp_async16(vs + i * VS + c * 4, A.v + ((tb + i) * A.H + h) * A.V + (long long)slab * VS + c * 4);
    }
    if (KIND == SKETCHSSM_KDA) {
        for (int x = tid; x < n * (KDIM / 4); x += nthr) {
            const int i = x >> 5, c = x & 31;
            cp_async16(as + i * KDIM + c * 4, A.a + ((tb + i) * A.H + h) * KDIM + c * 4);
        }
    } else if (tid < n) {
        cp_async4(as + tid, A.a + (tb + tid) * A.H + h);
    }
    if (KIND != SKETCHSSM_MAMBA2 && tid < n) cp_async4(bs + tid, A.beta + (tb + tid) * A.H + h);
}

template <int KIND>
__global__ void __launch_bounds__(PF_MAXT) prefill_kernel(const PrefillArgs A)
{
    extern __shared__ __align__(128) unsigned char psm[];
    const int V = A.V, VS = A.VS, nslab = V / VS, T = A.T;
    const PrefillCarve cv = prefill_carve(KIND, VS);
    float *ks_ = reinterpret_cast<float *>(psm + cv.k);
    float *vs_ = reinterpret_cast<float *>(psm + cv.v);
    float *as_ = reinterpret_cast<float *>(psm + cv.a);
    float *bs_ = reinterpret_cast<float *>(psm + cv.beta);
    const int da = KIND == SKETCHSSM_KDA ? KDIM : 1;

    const long long item = blockIdx.x;
    const long long bh = item / nslab;
    const int slab = (int)(item - bh * nslab);
    const long long b = bh / A.H;
    const int h = (int)(bh - b * A.H), qk = h / A.hpq;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ks = lane & 7, c4 = warp * 4 + (lane >> 3);
    const int nchunk = (T + PF_CHUNK - 1) / PF_CHUNK;

    issue_chunk<KIND>(A, b, h, qk, slab, 0, min(PF_CHUNK, T), ks_, vs_, as_, bs_);
    cp_async_commit();

    // the state slab, held in registers until the end of the prompt
    float *Sg = A.S + (bh * KDIM + 4 * ks) * V + (long long)slab * VS + c4 * 4;
    float4 s[16];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[4 * q + e] = *reinterpret_cast<const float4 *>(Sg + (long long)(32 * q + e) * V);

    for (int c = 0; c < nchunk; ++c) {
        const int st = c & 1;
        if (c + 1 < nchunk) {
            const int t1 = (c + 1) * PF_CHUNK;
            issue_chunk<KIND>(A, b, h, qk, slab, t1, min(PF_CHUNK, T - t1), ks_ + (st ^ 1) * PF_CHUNK * KDIM,
                              vs_ + (st ^ 1) * PF_CHUNK * VS, as_ + (st ^ 1) * PF_CHUNK * da,
                              bs_ + (st ^ 1) * PF_CHUNK);
        }
        cp_async_commit();
        cp_async_wait<1>();  // this thread's copies of chunk c have landed
        __syncthreads();     // and everyone's
        const float *kc = ks_ + st * PF_CHUNK * KDIM;
        const float *vc = vs_ + st * PF_CHUNK * VS;
        const float *ac = as_ + st * PF_CHUNK * da;
        const float *bc = bs_ + st * PF_CHUNK;
        const int n = min(PF_CHUNK, T - c * PF_CHUNK);
        if (KIND == SKETCHSSM_MAMBA2) {
            // the chunk at once: S <- P S + sum_i w_i k_i v_i^T with w_i = prod_{j>i} a_j
            // and P = prod_j a_j over the chunk's tokens, so that a token costs one FMA
            // per state element (its key is scaled by w_i first)
            float P = 1.f;
            for (int i = 0; i < n; ++i) P *= ac[i];
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                s[x].x *= P;
                s[x].y *= P;
                s[x].z *= P;
                s[x].w *= P;
            }
            float w = 1.f;  // w_i, walking the chunk newest first
            for (int i = n - 1; i >= 0; --i) {
                const float4 vv = lds4(vc + i * VS + c4 * 4);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 k4 = lds4(kc + i * KDIM + 4 * ks + 32 * q);
                    const float kk[4] = {w * k4.x, w * k4.y, w * k4.z, w * k4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) fma4(s[4 * q + e], kk[e], vv);
                }
                w *= ac[i];
            }
        } else {
            for (int i = 0; i < n; ++i) {
                float4 kq[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) kq[q] = lds4(kc + i * KDIM + 4 * ks + 32 * q);
                const float4 vv = lds4(vc + i * VS + c4 * 4);
                // d = S^T k for this column chunk, before the update
                float4 d = zero4();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    fma4(d, kq[q].x, s[4 * q + 0]);
                    fma4(d, kq[q].y, s[4 * q + 1]);
                    fma4(d, kq[q].z, s[4 * q + 2]);
                    fma4(d, kq[q].w, s[4 * q + 3]);
                }
                d = sum8_xor(d);
                const float bt = bc[i];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float kk[4] = {kq[q].x, kq[q].y, kq[q].z, kq[q].w};
                    float ak[4];
                    if (KIND == SKETCHSSM_KDA) {
                        const float4 a4 = lds4(ac + i * KDIM + 4 * ks + 32 * q);
                        ak[0] = a4.x;
                        ak[1] = a4.y;
                        ak[2] = a4.z;
                        ak[3] = a4.w;
                    } else {
                        ak[0] = ak[1] = ak[2] = ak[3] = ac[i];
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        // a (S - beta k d) + beta k v = a S + beta k (v - a d)
                        float4 &t = s[4 * q + e];
                        const float a_ = ak[e], kb = bt * kk[e];
                        t.x = fmaf(a_, t.x, kb * fmaf(-a_, d.x, vv.x));
                        t.y = fmaf(a_, t.y, kb * fmaf(-a_, d.y, vv.y));
                        t.z = fmaf(a_, t.z, kb * fmaf(-a_, d.z, vv.z));
                        t.w = fmaf(a_, t.w, kb * fmaf(-a_, d.w, vv.w));
                    }
                }
            }
        }
        __syncthreads();  // stage st is refilled by the next iteration's copies
    }

#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) st4(Sg + (long long)(32 * q + e) * V, s[4 * q + e]);
}

template <int KIND>
cudaError_t launch_kind(const PrefillArgs &a, cudaStream_t stream)
{
    const size_t smem = prefill_carve(KIND, a.VS).total;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long items = (long long)a.B * a.H * (a.V / a.VS);
    prefill_kernel<KIND><<<(unsigned)items, 2 * a.VS, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t stream)
{
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    switch (a.kind) {
    case SKETCHSSM_MAMBA2: return launch_kind<SKETCHSSM_MAMBA2>(a, stream);
    case SKETCHSSM_GDN: return launch_kind<SKETCHSSM_GDN>(a, stream);
    default: return launch_kind<SKETCHSSM_KDA>(a, stream);
    }
}

}  // namespace sk
