// Prefill handoff: the state after a prompt, the step before the decode path.  The
// paper's update is write-full (paper abstract: every state update reaches the full
// state); a prompt is taken in the same way, token after token: for every (batch row,
// head) apply t = 0 .. T-1 to S in place, S <- M_t S + beta_t k_t v_t^T (Mamba-2:
// M = a I, beta = 1; GDN: M = a (I - beta k k^T); KDA: M = diag(a) (I - beta k k^T)).
// The host then forms the sketch with the n = 0 flush.
//
// One CTA per (b, h, column slab of VS columns), 2 VS threads, the slab held in
// registers for the whole prompt, so S is read and written once however long the
// prompt.  The prompt comes through shared memory in chunks of PF_CHUNK tokens, double
// buffered with cp.async: chunk c + 1 is in flight while the CTA applies chunk c.  No
// thread waits on another CTA or on a flag: the only waits are cp.async groups and CTA
// barriers.
//   Mamba-2 prompts of at most 64 tokens with V a multiple of 16 up to 128 go to the
//   tcgen05 kernel (prefill_tcgen05.cu); the others:
//   Mamba-2 (prefill_tc_kernel): a chunk of n tokens is one contraction,
//     S <- P S + K^T (w o V), w_i = product of the later decays in the chunk, P of all,
//     on the tensor cores (mma.sync m16n8k8, tf32 operands split hi + lo, three
//     products, fp32 accumulators holding the state in the flush's layout).
//   GDN / KDA (prefill_kernel): thread (ks, c4) holds the float4 column chunk c4 of the
//     16 state rows 4 ks + 32 q + e, and applies the delta rule token by token; k^T S
//     is 3 xor-shuffle steps inside the warp.
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

// ---------------------------------------------------------------- Mamba-2 on the tensor cores
// Over a chunk of n <= 16 tokens the state update is S <- P S + K^T (w o V) (w_i = product
// of the later decays in the chunk, P of all of them): a contraction with inner dimension
// n.  It runs as mma.sync m16n8k8 with tf32 operands split x = hi + lo and the three
// products hi hi + hi lo + lo hi accumulated in fp32, the state held in the accumulators
// for the whole prompt.  Warp w owns columns 16 w .. 16 w + 15 of the slab for all 128
// rows: c[mt][nt][2 h + e] = state row srow(mt, g, h), column 16 w + 8 nt + 2 t + e
// (lane 4 g + t).

__device__ __forceinline__ void pf_split_tf32(float x, uint32_t &hi, uint32_t &lo)
{
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
    const float rest = x - __uint_as_float(hi);
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(rest));
}

__device__ __forceinline__ void pf_mma_tf32(float *d, const uint32_t *a, const uint32_t *b)
{
    asm(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// accumulator row 16 mt + g + 8 h <-> state row (a bijection of 0 .. 127)
__device__ __forceinline__ int pf_srow(int mt, int g, int h) { return 8 * g + 4 * h + 64 * (mt >> 2) + (mt & 3); }

struct TcCarve {
    size_t k, v, a, af, total;
    int vsp;  // padded value row: the B-fragment reads of a warp fall on 32 banks
    int ksp;  // padded key row: the fragment-building reads spread over 8 bank groups, not 4
};

__host__ __device__ inline TcCarve tc_carve(int VS)
{
    TcCarve c;
    c.vsp = VS + 8;
    c.ksp = KDIM + 4;
    size_t o = 0;
    c.k = o;
    o = pf_align(o + sizeof(float) * 2 * PF_CHUNK * (size_t)c.ksp);
    c.v = o;
    o = pf_align(o + sizeof(float) * 2 * PF_CHUNK * (size_t)c.vsp);
    c.a = o;  // decays [2][PF_CHUNK], then the chunk's w_i [PF_CHUNK] and P
    o = pf_align(o + sizeof(float) * (3 * PF_CHUNK + 1));
    c.af = o;  // [k-step][m-tile][hi, lo][lane][4]
    o = pf_align(o + sizeof(float) * (PF_CHUNK / 8) * 8 * 32 * 8);
    c.total = o;
    return c;
}

__global__ void __launch_bounds__(PF_MAXT, 3) prefill_tc_kernel(const PrefillArgs A)
{
    extern __shared__ __align__(128) unsigned char psm[];
    const int V = A.V, VS = A.VS, nslab = V / VS, T = A.T;
    const TcCarve cv = tc_carve(VS);
    float *ks_ = reinterpret_cast<float *>(psm + cv.k);
    float *vs_ = reinterpret_cast<float *>(psm + cv.v);
    float *as_ = reinterpret_cast<float *>(psm + cv.a);
    float *AF = reinterpret_cast<float *>(psm + cv.af);
    const int vsp = cv.vsp, ksp = cv.ksp;

    const long long item = blockIdx.x;
    const long long bh = item / nslab;
    const int slab = (int)(item - bh * nslab);
    const long long b = bh / A.H;
    const int h = (int)(bh - b * A.H), qk = h / A.hpq;
    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3, col0 = warp * 16;
    const int nchunk = (T + PF_CHUNK - 1) / PF_CHUNK;

    // copies of tokens t0 .. t0 + n - 1 into stage st
    auto issue = [&](int t0, int n, int st) {
        const long long tb = b * A.T + t0;
        float *kd = ks_ + st * PF_CHUNK * ksp, *vd = vs_ + st * PF_CHUNK * vsp, *ad = as_ + st * PF_CHUNK;
        for (int x = tid; x < n * (KDIM / 4); x += nthr) {
            const int i = x >> 5, c = x & 31;
            cp_async16(kd + i * ksp + c * 4, A.k + ((tb + i) * A.Hqk + qk) * KDIM + c * 4);
        }
        const int vq = VS / 4;
        for (int x = tid; x < n * vq; x += nthr) {
            const int i = x / vq, c = x - i * vq;
            cp_async16(vd + i * vsp + c * 4, A.v + ((tb + i) * A.H + h) * A.V + (long long)slab * VS + c * 4);
        }
        if (tid < n) cp_async4(ad + tid, A.a + (tb + tid) * A.H + h);
    };
    issue(0, min(PF_CHUNK, T), 0);
    cp_async_commit();

    float *Sg = A.S + bh * KDIM * V + (long long)slab * VS + col0 + 2 * t;
    float c[8][2][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const float2 lo = *reinterpret_cast<const float2 *>(Sg + (long long)pf_srow(mt, g, 0) * V + 8 * nt);
            const float2 hi = *reinterpret_cast<const float2 *>(Sg + (long long)pf_srow(mt, g, 1) * V + 8 * nt);
            c[mt][nt][0] = lo.x;
            c[mt][nt][1] = lo.y;
            c[mt][nt][2] = hi.x;
            c[mt][nt][3] = hi.y;
        }

    for (int ch = 0; ch < nchunk; ++ch) {
        const int st = ch & 1;
        cp_async_wait<0>();
        __syncthreads();  // chunk ch has landed; every warp is done with chunk ch - 1
        if (ch + 1 < nchunk) {
            const int t1 = (ch + 1) * PF_CHUNK;
            issue(t1, min(PF_CHUNK, T - t1), st ^ 1);
        }
        cp_async_commit();
        const int n = min(PF_CHUNK, T - ch * PF_CHUNK);
        const float *kt = ks_ + st * PF_CHUNK * ksp;
        const float *vt = vs_ + st * PF_CHUNK * vsp + col0 + g;
        const float *at = as_ + st * PF_CHUNK;
        // the keys' A fragments of this chunk, split hi / lo; tokens >= n are 0
        const int nkt = (n + 7) >> 3;
        for (int x = tid; x < nkt * 8 * 32 * 4; x += nthr) {
            const int comp = x & 3, ln = (x >> 2) & 31, mt = (x >> 7) & 7, k8 = x >> 10;
            const int tok = 8 * k8 + (ln & 3) + 4 * (comp >> 1);
            const float v = tok < n ? kt[tok * ksp + pf_srow(mt, ln >> 2, comp & 1)] : 0.f;
            uint32_t hi, lo;
            pf_split_tf32(v, hi, lo);
            float *f = AF + ((k8 * 8 + mt) * 64 + ln) * 4;  // hi, then lo 128 floats on
            f[comp] = __uint_as_float(hi);
            f[128 + comp] = __uint_as_float(lo);
        }
        // w_i = product of the decays after token i in the chunk (0 past the chunk), P of all
        float *wc = as_ + 2 * PF_CHUNK;
        if (warp == 0) {
            float x = lane < n ? at[lane] : 1.f;  // suffix products over the lanes
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, x, o);
                if (lane + o < 32) x *= y;
            }
            const float wl = __shfl_down_sync(0xffffffffu, x, 1);
            if (lane < PF_CHUNK) wc[lane] = lane < n ? (lane == 31 ? 1.f : wl) : 0.f;
            if (lane == 0) wc[PF_CHUNK] = x;
        }
        __syncthreads();  // the fragments and the weights are complete
        const float P = wc[PF_CHUNK];
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) c[mt][nt][e] *= P;
        for (int k0 = 0; k0 < n; k0 += 8) {
            const int i0 = k0 + t, i1 = k0 + t + 4;
            const float w0 = wc[i0], w1 = wc[i1];  // products of the decays after token i0, i1
            uint32_t bhf[2][2], blf[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const float v0 = i0 < n ? w0 * vt[i0 * vsp + 8 * nt] : 0.f;
                const float v1 = i1 < n ? w1 * vt[i1 * vsp + 8 * nt] : 0.f;
                pf_split_tf32(v0, bhf[nt][0], blf[nt][0]);
                pf_split_tf32(v1, bhf[nt][1], blf[nt][1]);
            }
            const float *af = AF + ((k0 >> 3) * 8 * 64 + lane) * 4;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const uint4 fh = *reinterpret_cast<const uint4 *>(af + mt * 64 * 4);
                const uint4 fl = *reinterpret_cast<const uint4 *>(af + mt * 64 * 4 + 128);
                const uint32_t ah[4] = {fh.x, fh.y, fh.z, fh.w}, al[4] = {fl.x, fl.y, fl.z, fl.w};
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    pf_mma_tf32(c[mt][nt], al, bhf[nt]);
                    pf_mma_tf32(c[mt][nt], ah, blf[nt]);
                    pf_mma_tf32(c[mt][nt], ah, bhf[nt]);
                }
            }
        }
    }

#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            *reinterpret_cast<float2 *>(Sg + (long long)pf_srow(mt, g, 0) * V + 8 * nt) =
                make_float2(c[mt][nt][0], c[mt][nt][1]);
            *reinterpret_cast<float2 *>(Sg + (long long)pf_srow(mt, g, 1) * V + 8 * nt) =
                make_float2(c[mt][nt][2], c[mt][nt][3]);
        }
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
    case SKETCHSSM_MAMBA2: {
        if (prefill_tcgen05_fits(a)) return launch_prefill_tcgen05(a, stream);
        const size_t smem = tc_carve(a.VS).total;
        cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const long long items = (long long)a.B * a.H * (a.V / a.VS);
        prefill_tc_kernel<<<(unsigned)items, 2 * a.VS, smem, stream>>>(a);
        return cudaGetLastError();
    }
    case SKETCHSSM_GDN: return launch_kind<SKETCHSSM_GDN>(a, stream);
    default: return launch_kind<SKETCHSSM_KDA>(a, stream);
    }
}

}  // namespace sk
