// Sketch decode and dense-read decode (one launch per decode step).
//
// Paper abstract (SketchSSM, newx.sg / mlsanity pages): a decode step "combines the
// sketch vectors with query-dependent coefficients to reconstruct the output
// without a full-state read"; the buffered keys and values since the last state
// update (ReplaySSM) are replayed exactly.  A head with a dense fallback (PyPI page,
// stage "allocate") reads the full state instead; the dense-read baseline does that
// for every head.
//
// One CTA per (work item, batch row).  A work item is either
//   - a group item: all sketch heads of one basis group (they share Omega_g and,
//     for Mamba-2 with group-shared B/C, the query and keys), or
//   - a dense item: one head whose base rows are its K state rows.
// Every head of an item contributes a list of rows, each a V-vector with a scalar
// coefficient: its base rows (sketch rows of Y, or state rows of S) and its n
// buffered value rows.  The output of the head is the weighted sum of its rows.
//
// Phase A computes the coefficients into shared memory:
//   Mamba-2: per q/k head s_i = k_i . q and u_m = Omega_g[m] . q (one warp per dot),
//            per head the suffix products w_i = prod_{j>i} a_j and decay_prod;
//            base coefficient decay_prod * u_m (sketch) or decay_prod * q_k (dense),
//            replay coefficient w_i s_i.
//   GDN/KDA: per head one warp walks the buffer newest first, x <- M_i^T x, with
//            replay coefficient beta_i (k_i . x); then q0 = x and the base
//            coefficients Omega_g[m] . q0 (sketch) or q0 itself (dense).
// Phase B streams every row once with 16-byte loads.  The item's row list is cut
// into `ns` contiguous chunks, one per slice of V/4 threads; each slice sums its
// chunk per head into a shared partial, and the partials of a head are added in
// slice order, so the result does not depend on scheduling.
// The step's own token is read from the inputs and appended at buffer slot pos
// (keys by the item that owns the first head of their q/k head).
#include "device_util.cuh"
#include "internal.cuh"

namespace sk {
namespace {

constexpr int DECODE_THREADS_TARGET = 320;
constexpr int DECODE_MAX_THREADS = 384;
constexpr int UNROLL = 8;

struct Carve {
    size_t hs, rstart, rbase, rneed, bptr, rinfo, coef, s, u, dp, q0, part, misc, total;
};

__host__ __device__ inline size_t take(size_t &o, size_t bytes)
{
    size_t r = o;
    o = (o + bytes + 15) & ~size_t(15);
    return r;
}

__host__ __device__ inline Carve carve(int Hg, int W, int cap, int max_rows, int ns, int V)
{
    Carve c;
    size_t o = 0;
    c.hs = take(o, sizeof(int) * Hg);
    c.rstart = take(o, sizeof(int) * (Hg + 1));
    c.rbase = take(o, sizeof(int) * Hg);
    c.rneed = take(o, sizeof(int) * Hg);
    c.bptr = take(o, sizeof(long long) * Hg);
    c.rinfo = take(o, sizeof(int) * max_rows);
    c.coef = take(o, sizeof(float) * max_rows);
    c.s = take(o, sizeof(float) * Hg * W);
    c.u = take(o, sizeof(float) * Hg * cap);
    c.dp = take(o, sizeof(float) * Hg);
    c.q0 = take(o, sizeof(float) * Hg * KDIM);
    c.part = take(o, sizeof(float) * (ns + Hg) * V);
    c.misc = take(o, sizeof(int) * 4);
    c.total = o;
    return c;
}

template <int KIND>
__global__ void __launch_bounds__(DECODE_MAX_THREADS)
decode_kernel(const DecodeArgs A)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const Carve cv = carve(A.Hg, A.W, A.cap, A.max_rows, A.ns, A.V);
    int *hs = reinterpret_cast<int *>(smem + cv.hs);
    int *rstart = reinterpret_cast<int *>(smem + cv.rstart);
    int *rbase = reinterpret_cast<int *>(smem + cv.rbase);
    int *rneed = reinterpret_cast<int *>(smem + cv.rneed);
    long long *bptr = reinterpret_cast<long long *>(smem + cv.bptr);
    int *rinfo = reinterpret_cast<int *>(smem + cv.rinfo);
    float *coef = reinterpret_cast<float *>(smem + cv.coef);
    float *s_dot = reinterpret_cast<float *>(smem + cv.s);
    float *u_dot = reinterpret_cast<float *>(smem + cv.u);
    float *dpv = reinterpret_cast<float *>(smem + cv.dp);
    float *q0s = reinterpret_cast<float *>(smem + cv.q0);
    float *part = reinterpret_cast<float *>(smem + cv.part);
    int *misc = reinterpret_cast<int *>(smem + cv.misc);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int b = blockIdx.y;
    const int item = A.dense_all ? -int(blockIdx.x) - 1 : A.work[blockIdx.x];
    const bool dense = item < 0;
    const int hd = -item - 1;                       // dense item: its head
    const int g = dense ? hd / A.Hg : item;         // basis group
    const int H = A.H, V = A.V, W = A.W, pos = A.pos, n = pos + 1;
    const int Hg = A.Hg, hpq = A.hpq, Hqk = A.Hqk;
    const int nch = dense ? 1 : Hg / hpq;          // q/k heads (chains) of a Mamba-2 item
    const float *base = dense ? A.S : A.Y;

    // ------------------------------------------------------------ item set-up
    if (warp == 0) {
        int h, rb;
        bool member;
        if (dense) {
            h = hd;
            member = lane == 0;
            rb = KDIM;
        } else {
            h = g * Hg + lane;
            const int r = (lane < Hg) ? __ldg(A.rank + h) : 0;
            member = r > 0;
            rb = r;
        }
        const unsigned mask = __ballot_sync(0xffffffffu, member);
        const int slot = __popc(mask & ((1u << lane) - 1u));
        const int rows = member ? rb + n : 0;
        int incl = rows;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane < Hg) rneed[lane] = -1;
        __syncwarp();
        if (member) {
            hs[slot] = h;
            rbase[slot] = rb;
            rstart[slot] = incl - rows;
            bptr[slot] = dense ? ((long long)b * H + h) * KDIM * V
                               : ((long long)b * A.rtot + __ldg(A.off + h)) * V;
            if (KIND == SKETCHSSM_MAMBA2) atomicMax(&rneed[dense ? 0 : (h - g * Hg) / hpq], dense ? 0 : rb);
        }
        if (lane == 31) {
            const int nh = __popc(mask);
            misc[0] = nh;
            misc[1] = incl;
            rstart[nh] = incl;
        }
    }
    __syncthreads();
    const int nh = misc[0], total = misc[1];
    for (int hl = warp; hl < nh; hl += nwarps) {
        const int rows = rbase[hl] + n, r0 = rstart[hl];
        for (int j = lane; j < rows; j += 32) rinfo[r0 + j] = (hl << 16) | j;
    }

    // ------------------------------------------------------------ phase A
    if (KIND == SKETCHSSM_MAMBA2) {
        // dot products of one warp each: chain c has n key dots and rneed[c] basis dots
        const int cnt = (lane < nch && rneed[lane] >= 0) ? n + rneed[lane] : 0;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const int start = incl - cnt;
        const int ntask = __shfl_sync(0xffffffffu, incl, 31);
        for (int t = warp; t < ntask; t += nwarps) {
            const unsigned hit = __ballot_sync(0xffffffffu, cnt > 0 && start <= t && t < start + cnt);
            const int c = __ffs(hit) - 1;
            const int idx = t - __shfl_sync(0xffffffffu, start, c);
            const int qk = dense ? hd / hpq : (g * Hg) / hpq + c;
            const long long qrow = (long long)b * Hqk + qk;
            const float4 qv = ldg4(A.q + qrow * KDIM + lane * 4);
            float4 vec;
            if (idx < n) {
                vec = (idx == pos) ? ldg4(A.k + qrow * KDIM + lane * 4)
                                   : ldg4(A.kbuf + (qrow * W + idx) * KDIM + lane * 4);
            } else {
                vec = ldg4(A.omega + ((long long)g * A.Rb + (idx - n)) * KDIM + lane * 4);
            }
            const float d = warp_sum(dot4(qv, vec));
            if (lane == 0) {
                if (idx < n) s_dot[c * W + idx] = d;
                else u_dot[c * A.cap + (idx - n)] = d;
            }
            if (idx == pos) {
                // this item writes the key if it handles the first head of the q/k head
                const int h0 = qk * hpq;
                const bool owner = dense ? (hd == h0) : (__ldg(A.rank + h0) > 0);
                if (owner) st4(A.kbuf + (qrow * W + pos) * KDIM + lane * 4, vec);
            }
        }
        __syncthreads();
        if (tid < nh) {
            const int h = hs[tid];
            const int c = dense ? 0 : (h - g * Hg) / hpq;
            const long long bh = (long long)b * H + h;
            const int r0 = rstart[tid] + rbase[tid];
            float dp = 1.f;
            for (int i = n - 1; i >= 0; --i) {
                const float ai = (i == pos) ? __ldg(A.a + bh) : __ldg(A.abuf + bh * W + i);
                coef[r0 + i] = dp * s_dot[c * W + i];
                dp *= ai;
            }
            dpv[tid] = dp;
            A.abuf[bh * W + pos] = __ldg(A.a + bh);
        }
        __syncthreads();
        for (int e = tid; e < total; e += blockDim.x) {
            const int info = rinfo[e], hl = info >> 16, j = info & 0xffff;
            if (j >= rbase[hl]) continue;
            if (dense) {
                coef[e] = dpv[0] * __ldg(A.q + ((long long)b * Hqk + hd / hpq) * KDIM + j);
            } else {
                const int c = (hs[hl] - g * Hg) / hpq;
                coef[e] = dpv[hl] * u_dot[c * A.cap + j];
            }
        }
    } else {
        // GDN / KDA: one warp per head walks the buffer newest first
        for (int hl = warp; hl < nh; hl += nwarps) {
            const int h = hs[hl], qk = h / hpq;
            const long long bh = (long long)b * H + h;
            const long long qrow = (long long)b * Hqk + qk;
            float4 x = ldg4(A.q + qrow * KDIM + lane * 4);
            const int r0 = rstart[hl] + rbase[hl];
            for (int i = n - 1; i >= 0; --i) {
                const bool cur = (i == pos);
                const float4 kv = cur ? ldg4(A.k + qrow * KDIM + lane * 4)
                                      : ldg4(A.kbuf + (qrow * W + i) * KDIM + lane * 4);
                const float bi = cur ? __ldg(A.beta + bh) : __ldg(A.bbuf + bh * W + i);
                const float s1 = warp_sum(dot4(kv, x));
                if (lane == 0) coef[r0 + i] = bi * s1;
                if (KIND == SKETCHSSM_GDN) {
                    const float ai = cur ? __ldg(A.a + bh) : __ldg(A.abuf + bh * W + i);
                    const float t = bi * s1;
                    x.x = ai * fmaf(-t, kv.x, x.x);
                    x.y = ai * fmaf(-t, kv.y, x.y);
                    x.z = ai * fmaf(-t, kv.z, x.z);
                    x.w = ai * fmaf(-t, kv.w, x.w);
                    if (cur && lane == 0) A.abuf[bh * W + pos] = ai;
                } else {
                    const float4 av = cur ? ldg4(A.a + bh * KDIM + lane * 4)
                                          : ldg4(A.abuf + (bh * W + i) * KDIM + lane * 4);
                    const float4 xa = make_float4(av.x * x.x, av.y * x.y, av.z * x.z, av.w * x.w);
                    const float t = bi * warp_sum(dot4(kv, xa));
                    x.x = fmaf(-t, kv.x, xa.x);
                    x.y = fmaf(-t, kv.y, xa.y);
                    x.z = fmaf(-t, kv.z, xa.z);
                    x.w = fmaf(-t, kv.w, xa.w);
                    if (cur) st4(A.abuf + (bh * W + pos) * KDIM + lane * 4, av);
                }
                if (cur) {
                    if (h == qk * hpq) st4(A.kbuf + (qrow * W + pos) * KDIM + lane * 4, kv);
                    if (lane == 0) A.bbuf[bh * W + pos] = bi;
                }
            }
            st4(q0s + hl * KDIM + lane * 4, x);
        }
        __syncthreads();
        if (dense) {
            for (int j = tid; j < KDIM; j += blockDim.x) coef[j] = q0s[j];
        } else {
            for (int e = warp; e < total; e += nwarps) {
                const int info = rinfo[e], hl = info >> 16, j = info & 0xffff;
                if (j >= rbase[hl]) continue;  // warp-uniform
                const float4 om = ldg4(A.omega + ((long long)g * A.Rb + j) * KDIM + lane * 4);
                const float d = warp_sum(dot4(om, lds4(q0s + hl * KDIM + lane * 4)));
                if (lane == 0) coef[e] = d;
            }
        }
    }
    __syncthreads();

    // ------------------------------------------------------------ phase B
    const int V4 = V >> 2;
    const int ns = A.ns;
    const int chunk = (total + ns - 1) / ns;
    const int sl = tid / V4, c4 = tid - sl * V4;
    if (sl < ns) {
        const int e0 = sl * chunk;
        const int e1 = min(e0 + chunk, total);
        float4 acc = zero4();
        int curh = -1;
        for (int e = e0; e < e1; e += UNROLL) {
            float4 xv[UNROLL];
            float cf[UNROLL];
            int hv[UNROLL];
            float *app[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                hv[u] = -1;
                app[u] = nullptr;
                const int ee = e + u;
                if (ee < e1) {
                    const int info = rinfo[ee], hl = info >> 16, j = info & 0xffff;
                    const int rb = rbase[hl];
                    const float *src;
                    if (j < rb) {
                        src = base + bptr[hl] + (long long)j * V;
                    } else {
                        const int i = j - rb;
                        const long long bh = (long long)b * H + hs[hl];
                        if (i == pos) {
                            src = A.v + bh * V;
                            app[u] = A.vbuf + (bh * W + pos) * V + c4 * 4;
                        } else {
                            src = A.vbuf + (bh * W + i) * V;
                        }
                    }
                    xv[u] = ldg4(src + c4 * 4);
                    cf[u] = coef[ee];
                    hv[u] = hl;
                }
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u)
                if (app[u]) st4(app[u], xv[u]);
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                if (hv[u] < 0) continue;
                if (hv[u] != curh) {
                    if (curh >= 0) st4(part + (sl + curh) * V + c4 * 4, acc);
                    acc = zero4();
                    curh = hv[u];
                }
                fma4(acc, cf[u], xv[u]);
            }
        }
        if (curh >= 0) st4(part + (sl + curh) * V + c4 * 4, acc);
    }
    __syncthreads();
    for (int o = tid; o < nh * V4; o += blockDim.x) {
        const int hl = o / V4, cc = o - hl * V4;
        const int s0 = rstart[hl] / chunk, s1 = (rstart[hl + 1] - 1) / chunk;
        float4 sum = zero4();
        for (int s = s0; s <= s1; ++s) {
            const float4 p = lds4(part + (s + hl) * V + cc * 4);
            sum.x += p.x;
            sum.y += p.y;
            sum.z += p.z;
            sum.w += p.w;
        }
        st4(A.y + ((long long)b * H + hs[hl]) * V + cc * 4, sum);
    }
}

template <int KIND>
cudaError_t launch_kind(const DecodeArgs &a, cudaStream_t stream)
{
    int ns = 0;
    const int threads = decode_threads(a.V, &ns);
    const size_t smem = decode_smem_bytes(a);
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<KIND>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(a.dense_all ? a.H : a.n_work, a.B);
    decode_kernel<KIND><<<grid, threads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

int decode_threads(int V, int *ns_out)
{
    const int V4 = V / 4;
    int ns = DECODE_THREADS_TARGET / V4;
    if (ns < 1) ns = 1;
    if (ns_out) *ns_out = ns;
    return ((ns * V4 + 31) / 32) * 32;
}

size_t decode_smem_bytes(const DecodeArgs &a)
{
    return carve(a.Hg, a.W, a.cap, a.max_rows, a.ns, a.V).total;
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream)
{
    if (a.B == 0 || (a.dense_all ? a.H : a.n_work) == 0) return cudaSuccess;
    switch (a.kind) {
    case SKETCHSSM_MAMBA2: return launch_kind<SKETCHSSM_MAMBA2>(a, stream);
    case SKETCHSSM_GDN: return launch_kind<SKETCHSSM_GDN>(a, stream);
    default: return launch_kind<SKETCHSSM_KDA>(a, stream);
    }
}

}  // namespace sk
