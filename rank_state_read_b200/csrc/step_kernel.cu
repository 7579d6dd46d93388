// The standard per-step recurrent decode: the baseline the SketchSSM paper measures its
// speedup against (paper abstract: standard decoding reads and updates the full state
// for every token).  For every (batch row, head): apply the step's token to the state,
// S <- M S + beta k v^T (Mamba-2: M = a I, beta = 1; GDN: M = a (I - beta k k^T); KDA:
// M = diag(a) (I - beta k k^T)), write S back and read it after the update, y = S^T q.
// No buffer and no sketch: every step moves 2 K V 4 bytes per (b, h).
//
// One CTA per (b, h, column slab of VS columns), 2 VS threads, several CTAs per SM.
// Thread (ks, c4) holds the float4 column chunk c4 of the 16 state rows
// 4 ks + 32 q + e (q, e < 4), so the reductions over k (the delta rule's k^T S and the
// read S^T q) are 3 xor-shuffle steps inside the warp and the float4 reads of k, q and
// the KDA decays by the 8 row slices are 128 consecutive bytes.  Warp 0 brings the
// state slab (32 chunks of 4 rows, each chunk padded by 4 floats: conflict-free reads)
// and the token's rows in with TMA bulk copies on one mbarrier; the wait is bounded.
#include "device_util.cuh"
#include "internal.cuh"
#include "ptx_util.cuh"

namespace sk {
namespace {

constexpr int STEP_MAXT = 160;  // slabs of at most 80 columns

struct StepCarve {
    size_t bar, S, k, q, a, v, total;
};

__host__ __device__ inline size_t step_align(size_t x) { return (x + 127) & ~size_t(127); }

__host__ __device__ inline StepCarve step_carve(int kind, int VS)
{
    StepCarve c;
    size_t o = 0;
    c.bar = o;
    o = step_align(o + 16);
    c.S = o;
    o = step_align(o + sizeof(float) * 32 * (size_t)(4 * VS + 4));
    c.k = o;
    o = step_align(o + sizeof(float) * KDIM);
    c.q = o;
    o = step_align(o + sizeof(float) * KDIM);
    c.a = o;
    o = step_align(o + (kind == SKETCHSSM_KDA ? sizeof(float) * KDIM : 0));
    c.v = o;
    o = step_align(o + sizeof(float) * (size_t)VS);
    c.total = o;
    return c;
}

// Mamba-2 fits four CTAs of 160 threads per SM; the delta rule's extra registers (the
// erase term) three
template <int KIND>
__global__ void __launch_bounds__(STEP_MAXT, KIND == SKETCHSSM_MAMBA2 ? 4 : 3) step_kernel(const StepArgs A)
{
    extern __shared__ __align__(128) unsigned char ssm[];
    const int V = A.V, VS = A.VS, nslab = V / VS;
    const StepCarve cv = step_carve(KIND, VS);
    uint64_t *bar = reinterpret_cast<uint64_t *>(ssm + cv.bar);
    float *Sb = reinterpret_cast<float *>(ssm + cv.S);
    float *ks_ = reinterpret_cast<float *>(ssm + cv.k);
    float *qs = reinterpret_cast<float *>(ssm + cv.q);
    float *as = reinterpret_cast<float *>(ssm + cv.a);
    float *vs = reinterpret_cast<float *>(ssm + cv.v);

    const long long item = blockIdx.x;
    const long long bh = item / nslab;
    const int slab = (int)(item - bh * nslab);
    const int b = (int)(bh / A.H), h = (int)(bh - (long long)b * A.H);
    const long long qrow = (long long)b * A.Hqk + h / A.hpq;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ks = lane & 7, c4 = warp * 4 + (lane >> 3);

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    const float *Sg = A.S + bh * KDIM * V + (long long)slab * VS;
    if (warp == 0) {
        if (lane == 0) {
            const uint32_t bytes =
                (uint32_t)(4 * (KDIM * VS + 2 * KDIM + VS + (KIND == SKETCHSSM_KDA ? KDIM : 0)));
            mbar_arrive_expect_tx(bar, bytes);
        }
        __syncwarp();
        float *dst = Sb + (size_t)lane * (4 * VS + 4);
        if (nslab == 1) {  // 4 state rows are 4 V contiguous floats
            bulk_copy_g2s(dst, Sg + (long long)lane * 4 * V, (uint32_t)(16 * VS), bar);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                bulk_copy_g2s(dst + e * VS, Sg + (long long)(lane * 4 + e) * V, (uint32_t)(4 * VS), bar);
        }
        if (lane == 0) bulk_copy_g2s(ks_, A.k + qrow * KDIM, KDIM * 4, bar);
        if (lane == 1) bulk_copy_g2s(qs, A.q + qrow * KDIM, KDIM * 4, bar);
        if (lane == 2) bulk_copy_g2s(vs, A.v + bh * V + (long long)slab * VS, (uint32_t)(VS * 4), bar);
        if (KIND == SKETCHSSM_KDA && lane == 3) bulk_copy_g2s(as, A.a + bh * KDIM, KDIM * 4, bar);
    }
    const float at = KIND == SKETCHSSM_KDA ? 1.f : __ldg(A.a + bh);
    const float bt = KIND == SKETCHSSM_MAMBA2 ? 1.f : __ldg(A.beta + bh);

    // bounded wait: past the plan's limit it is recorded and continued to the default
    bool ok = mbar_wait_bounded(bar, 0, A.wait_limit);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) atomicOr(A.status, SK_STATUS_STEP_TIMEOUT);
        ok = mbar_wait_bounded(bar, 0, DEFAULT_WAIT_CYCLES);
        if (__syncthreads_or(!ok)) {
            // give up: let the copies still in flight land (bounded) before the CTA exits
            if (tid == 0) mbar_wait_bounded(bar, 0, DEFAULT_WAIT_CYCLES);
            __syncthreads();
            return;
        }
    }

    float4 s[16];
    {
        const float *sb = Sb + (size_t)ks * (4 * VS + 4) + c4 * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[4 * q + e] = lds4(sb + (size_t)q * 8 * (4 * VS + 4) + e * VS);
    }
    float4 kq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) kq[q] = lds4(ks_ + 4 * ks + 32 * q);
    const float4 vv = lds4(vs + c4 * 4);

    if (KIND == SKETCHSSM_MAMBA2) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float kk[4] = {kq[q].x, kq[q].y, kq[q].z, kq[q].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float4 &t = s[4 * q + e];
                t.x = fmaf(at, t.x, kk[e] * vv.x);
                t.y = fmaf(at, t.y, kk[e] * vv.y);
                t.z = fmaf(at, t.z, kk[e] * vv.z);
                t.w = fmaf(at, t.w, kk[e] * vv.w);
            }
        }
    } else {
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
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float kk[4] = {kq[q].x, kq[q].y, kq[q].z, kq[q].w};
            float ak[4] = {at, at, at, at};
            if (KIND == SKETCHSSM_KDA) {
                const float4 a4 = lds4(as + 4 * ks + 32 * q);
                ak[0] = a4.x;
                ak[1] = a4.y;
                ak[2] = a4.z;
                ak[3] = a4.w;
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

    float *Sw = A.S + (bh * KDIM + 4 * ks) * V + (long long)slab * VS + c4 * 4;
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) st4(Sw + (long long)(32 * q + e) * V, s[4 * q + e]);

    // y = S^T q, read after the update
    float4 p = zero4();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 qq = lds4(qs + 4 * ks + 32 * q);
        fma4(p, qq.x, s[4 * q + 0]);
        fma4(p, qq.y, s[4 * q + 1]);
        fma4(p, qq.z, s[4 * q + 2]);
        fma4(p, qq.w, s[4 * q + 3]);
    }
    p = sum8_xor(p);
    if (ks == 0) st4(A.y + bh * V + (long long)slab * VS + c4 * 4, p);
}

template <int KIND>
cudaError_t launch_kind(const StepArgs &a, cudaStream_t stream)
{
    const size_t smem = step_carve(KIND, a.VS).total;
    cudaError_t e = cudaFuncSetAttribute(step_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long items = (long long)a.B * a.H * (a.V / a.VS);
    step_kernel<KIND><<<(unsigned)items, 2 * a.VS, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

int step_slab(int V)
{
    if (V <= 80) return V;
    for (int vs = 64; vs >= 16; vs -= 16)
        if (V % vs == 0) return vs;
    return 16;
}

cudaError_t launch_step(const StepArgs &a, cudaStream_t stream)
{
    if (a.B == 0) return cudaSuccess;
    switch (a.kind) {
    case SKETCHSSM_MAMBA2: return launch_kind<SKETCHSSM_MAMBA2>(a, stream);
    case SKETCHSSM_GDN: return launch_kind<SKETCHSSM_GDN>(a, stream);
    default: return launch_kind<SKETCHSSM_KDA>(a, stream);
    }
}

}  // namespace sk
