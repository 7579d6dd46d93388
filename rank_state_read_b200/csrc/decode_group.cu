// Mamba-2 sketch decode in one launch: one CTA per (basis group, batch row).
//
// Paper abstract (SketchSSM, newx.sg / mlsanity pages): a decode step rebuilds each
// head's output from its r sketch rows, weighted by coefficients computed from the
// query, plus the exact replay of the keys and values buffered since the last state
// update (ReplaySSM); a head with a dense fallback (PyPI page, stage "allocate") reads
// its full state instead.  For Mamba-2 with scalar decay a and the q/k head of head h:
//   s_i = k_i . q (i <= pos, k_pos the step's key),  u_m = Omega_g[m] . q,
//   w_i = prod_{j > i} a_j,  P = prod_j a_j,
//   y_h = sum_i w_i s_i v_i + P sum_{m < r_h} u_m Y_h[m]     (sketch head)
//   y_h = sum_i w_i s_i v_i + P sum_{k < K} q_k S_h[k]      (dense head).
//
// Every output is a weighted sum of rows of V floats.  The rows a CTA needs form two
// lists, streamed through a ring of shared-memory stages by bulk (TMA) copies, one
// mbarrier per stage:
//   value list: per head of the group its n = pos + 1 value rows (pos from vbuf, the
//               step's from v); its addresses need nothing but pos, so its first
//               stages are issued before the CTA has read anything;
//   base list:  the group's block of Y (the sketch heads' rows are contiguous), then
//               the full state of each dense head of the group.
// While the first stages land, the CTA forms the products it needs in shared memory
// (one warp per dot product, lanes over k, loads batched four dots deep) and the
// per-head decay weights.  Thread (head, column chunk) then sums its head's rows in
// list order (deterministic), writes y, and appends the step's value; the step's key
// and decay are appended during the products.  No scratch memory, no second launch.
//
// Every wait on a stage is bounded by the plan's limit (recorded, then continued up to
// DEFAULT_WAIT_CYCLES); a CTA that gives up lets the copies it issued land (bounded)
// before it exits.
#include "device_util.cuh"
#include "internal.cuh"
#include "ptx_util.cuh"

namespace sk {
namespace {

constexpr int DG_MAX_THREADS = 512;
constexpr int DG_BATCH = 4;  // dot products per warp in flight

// ring of stages: DG_STAGES slots of DG_STAGE_BYTES (rounded down to whole rows)
#ifndef DG_STAGES
#define DG_STAGES 2
#endif
#ifndef DG_STAGE_BYTES
#define DG_STAGE_BYTES (40 * 1024)
#endif

struct DgCarve {
    size_t bar, meta, qs, as, ph, dots, wv, stage, total;
};

__host__ __device__ inline size_t dg_take(size_t &o, size_t bytes)
{
    const size_t r = o;
    o = (o + bytes + 127) & ~size_t(127);
    return r;
}

__host__ __device__ inline DgCarve dg_carve(int V, int W, int Hg, int nq, int cap, int nst, int sb)
{
    DgCarve c;
    size_t o = 0;
    c.bar = dg_take(o, 8 * (size_t)nst);
    c.meta = dg_take(o, sizeof(int) * (4 * MAX_HG + 4 + MAX_HG));
    c.qs = dg_take(o, sizeof(float) * (size_t)nq * KDIM);
    c.as = dg_take(o, sizeof(float) * (size_t)Hg * W);
    c.ph = dg_take(o, sizeof(float) * MAX_HG);
    c.dots = dg_take(o, sizeof(float) * (size_t)nq * (W + cap));
    c.wv = dg_take(o, sizeof(float) * (size_t)Hg * W);
    c.stage = dg_take(o, sizeof(float) * (size_t)nst * sb * V);
    c.total = o;
    return c;
}

template <int MAXP>
__global__ void __launch_bounds__(DG_MAX_THREADS)
decode_group_kernel(const DecodeArgs A, const int nst, const int sb)
{
    extern __shared__ __align__(128) unsigned char dsm[];
    const int G = A.G;
    const int b = blockIdx.x / G, g = blockIdx.x - b * G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
    // buffer position of this row (per-row positions: out of range is recorded, row left alone)
    int pos = A.pos;
    if (A.row_pos) {
        pos = __ldg(A.row_pos + b);
        if (pos < 0 || pos >= A.W) {
            if (tid == 0) atomicOr(A.status, SK_STATUS_BAD_ROW);
            return;
        }
    }
    const int H = A.H, V = A.V, W = A.W, Hg = A.Hg, hpq = A.hpq, n = pos + 1, cap = A.cap;
    const int h0 = g * Hg, nq = Hg / hpq, q0 = h0 / hpq;
    const DgCarve cv = dg_carve(V, W, Hg, nq, cap, nst, sb);
    uint64_t *bar = reinterpret_cast<uint64_t *>(dsm + cv.bar);
    int *m_rank = reinterpret_cast<int *>(dsm + cv.meta);  // rank, or -1 for a dense head
    int *m_rbs = m_rank + MAX_HG;                          // first row in the group's Y block
    int *m_didx = m_rank + 2 * MAX_HG;                     // index among the group's dense heads
    int *m_dh = m_rank + 3 * MAX_HG;                       // dense heads, in order
    int *m_tot = m_rank + 4 * MAX_HG;                      // {RY, nd, off[h0]}
    int *m_nu = m_tot + 4;                                 // basis rows needed per q/k head
    float *qs = reinterpret_cast<float *>(dsm + cv.qs);
    float *as_ = reinterpret_cast<float *>(dsm + cv.as);
    float *Ph = reinterpret_cast<float *>(dsm + cv.ph);
    float *dots = reinterpret_cast<float *>(dsm + cv.dots);
    float *wv = reinterpret_cast<float *>(dsm + cv.wv);
    float *stage = reinterpret_cast<float *>(dsm + cv.stage);
    const int dstride = W + cap;
    const long long rowq = (long long)b * A.Hqk + q0;  // first q/k row of the group
    const int nvr = Hg * n;                            // value rows
    const int nvs = (nvr + sb - 1) / sb;               // value stages

    // bulk copies of value-list rows [s0, s1) into ring slot k % nst (warp 0, lane per head)
    auto issue_value = [&](int k) {
        const int st = k % nst, s0 = k * sb, s1 = min(nvr, s0 + sb);
        float *dst = stage + (size_t)st * sb * V;
        if (lane == 0) mbar_arrive_expect_tx(bar + st, (uint32_t)((s1 - s0) * V * 4));
        __syncwarp();
        if (lane < Hg) {
            const long long bh = (long long)b * H + h0 + lane;
            const int lo = lane * n;
            const int a0 = max(lo, s0), a1 = min(lo + pos, s1);  // buffered rows 0 .. pos-1
            if (a0 < a1)
                bulk_copy_g2s(dst + (size_t)(a0 - s0) * V, A.vbuf + (bh * W + (a0 - lo)) * V,
                              (uint32_t)((a1 - a0) * V * 4), bar + st);
            if (lo + pos >= s0 && lo + pos < s1)  // the step's value
                bulk_copy_g2s(dst + (size_t)(lo + pos - s0) * V, A.v + bh * V, (uint32_t)(V * 4), bar + st);
        }
    };

    if (warp == 0) {
        const int r = lane < Hg ? __ldg(A.rank + h0 + lane) : 0;  // in flight with the first copies
        const int offg = __ldg(A.off + h0);
        if (lane == 0) {
            for (int s = 0; s < nst; ++s) mbar_init(bar + s, 1);
            mbar_fence_init();
        }
        __syncwarp();
        for (int k = 0; k < nvs && k < nst; ++k) issue_value(k);
        const bool dense = lane < Hg && r <= 0;
        int incl = (lane < Hg && !dense) ? r : 0, dinc = dense ? 1 : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, incl, o), y = __shfl_up_sync(0xffffffffu, dinc, o);
            if (lane >= o) {
                incl += x;
                dinc += y;
            }
        }
        if (lane < Hg) {
            m_rank[lane] = dense ? -1 : r;
            m_rbs[lane] = dense ? 0 : incl - r;
            m_didx[lane] = dense ? dinc - 1 : -1;
            if (dense) m_dh[dinc - 1] = h0 + lane;
        }
        if (lane == 31) {
            m_tot[0] = incl;  // sketch rows of the group
            m_tot[1] = dinc;  // dense heads of the group
            m_tot[2] = offg;
        }
        __syncwarp();
        if (lane < nq) {  // basis rows needed by the heads of each q/k head
            int nu = 0;
            for (int j = 0; j < hpq; ++j) nu = max(nu, m_rank[lane * hpq + j]);
            m_nu[lane] = nu;
        }
    } else {
        // the group's queries; the members' decays (the step's appended at pos)
        for (int x = tid - 32; x < nq * (KDIM / 4); x += blockDim.x - 32) {
            const int qi = x >> 5, c = x & 31;
            st4(qs + qi * KDIM + c * 4, ldg4(A.q + (rowq + qi) * KDIM + c * 4));
        }
        for (int x = tid - 32; x < Hg * n; x += blockDim.x - 32) {
            const int hl = x / n, i = x - hl * n;
            const long long bh = (long long)b * H + h0 + hl;
            const float av = (i == pos) ? __ldg(A.a + bh) : __ldg(A.abuf + bh * W + i);
            as_[hl * W + i] = av;
            if (i == pos) A.abuf[bh * W + pos] = av;
        }
        // key products s_i = k_i . q; the step's key is appended at slot pos
        const int total = nq * n;
        for (int j0 = warp - 1; j0 < total; j0 += (nwarp - 1) * DG_BATCH) {
            float4 rv[DG_BATCH], qv[DG_BATCH];
#pragma unroll
            for (int u = 0; u < DG_BATCH; ++u) {
                const int j = j0 + u * (nwarp - 1);
                rv[u] = qv[u] = zero4();
                if (j < total) {
                    const int qi = j / n, e = j - qi * n;
                    const long long qrow = rowq + qi;
                    rv[u] = ldg4((e == pos ? A.k + qrow * KDIM : A.kbuf + (qrow * W + e) * KDIM) + lane * 4);
                    qv[u] = ldg4(A.q + qrow * KDIM + lane * 4);
                }
            }
#pragma unroll
            for (int u = 0; u < DG_BATCH; ++u) {
                const int j = j0 + u * (nwarp - 1);
                if (j >= total) break;
                const int qi = j / n, e = j - qi * n;
                const float d = warp_sum(dot4(rv[u], qv[u]));
                if (lane == 0) dots[qi * dstride + e] = d;
                if (e == pos) st4(A.kbuf + ((rowq + qi) * W + pos) * KDIM + lane * 4, rv[u]);
            }
        }
    }
    __syncthreads();
    const int RY = m_tot[0], nd = m_tot[1];
    const int nbr = RY + KDIM * nd;                // base rows
    const int ns = nvs + (nbr + sb - 1) / sb;      // stages in all
    const long long ybase = (long long)b * A.rtot + m_tot[2];

    // bulk copies of base-list rows into ring slot k % nst (warp 0)
    auto issue_base = [&](int k) {
        const int st = k % nst, s0 = (k - nvs) * sb, s1 = min(nbr, s0 + sb);
        float *dst = stage + (size_t)st * sb * V;
        if (lane == 0) {
            mbar_arrive_expect_tx(bar + st, (uint32_t)((s1 - s0) * V * 4));
            if (s0 < RY)
                bulk_copy_g2s(dst, A.Y + (ybase + s0) * V, (uint32_t)((min(RY, s1) - s0) * V * 4), bar + st);
        }
        __syncwarp();
        if (lane < nd) {
            const int lo = RY + KDIM * lane, a0 = max(lo, s0), a1 = min(lo + KDIM, s1);
            if (a0 < a1)
                bulk_copy_g2s(dst + (size_t)(a0 - s0) * V,
                              A.S + (((long long)b * H + m_dh[lane]) * KDIM + (a0 - lo)) * V,
                              (uint32_t)((a1 - a0) * V * 4), bar + st);
        }
    };
    if (warp == 0)
        for (int k = nvs; k < ns && k < nst; ++k) issue_base(k);

    // basis products u_m = Omega_g[m] . q for m below each q/k head's largest sketch rank
    {
        int nu_all = 0;
        for (int qi = 0; qi < nq; ++qi) nu_all = max(nu_all, m_nu[qi]);
        const int total = nq * nu_all;
        const float *og = A.omega + (long long)g * A.Rb * KDIM;
        for (int j0 = warp; j0 < total; j0 += nwarp * DG_BATCH) {
            float4 rv[DG_BATCH], qv[DG_BATCH];
#pragma unroll
            for (int u = 0; u < DG_BATCH; ++u) {
                const int j = j0 + u * nwarp;
                rv[u] = qv[u] = zero4();
                if (j < total) {
                    const int qi = j / nu_all, m = j - qi * nu_all;
                    if (m < m_nu[qi]) {
                        rv[u] = ldg4(og + (long long)m * KDIM + lane * 4);
                        qv[u] = lds4(qs + qi * KDIM + lane * 4);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < DG_BATCH; ++u) {
                const int j = j0 + u * nwarp;
                if (j >= total) break;
                const int qi = j / nu_all, m = j - qi * nu_all;
                const float d = warp_sum(dot4(rv[u], qv[u]));
                if (lane == 0 && m < m_nu[qi]) dots[qi * dstride + W + m] = d;
            }
        }
    }
    // per head: decay weights of the value rows w_i s_i (newest first) and P
    if (tid < Hg) {
        const int hl = tid, qi = (h0 + hl) / hpq - q0;
        float w = 1.f;
        for (int i = n - 1; i >= 0; --i) {
            wv[hl * W + i] = w * dots[qi * dstride + i];
            w *= as_[hl * W + i];
        }
        Ph[hl] = w;
    }
    __syncthreads();

    // stream the stages; thread owns (head, column chunk) pairs tid + p * blockDim.x
    const int V4 = V >> 2, npair = Hg * V4;
    float4 acc[MAXP];
#pragma unroll
    for (int p = 0; p < MAXP; ++p) acc[p] = zero4();
    for (int k = 0; k < ns; ++k) {
        const int st = k % nst;
        const uint32_t par = (uint32_t)((k / nst) & 1);
        bool got = mbar_wait_bounded(bar + st, par, A.wait_limit);
        if (__syncthreads_or(!got)) {
            if (tid == 0) atomicOr(A.status, SK_STATUS_DECODE_TIMEOUT);
            got = mbar_wait_bounded(bar + st, par, DEFAULT_WAIT_CYCLES);
            if (__syncthreads_or(!got)) {
                // give up: let the copies still in flight land before the CTA exits
                if (tid == 0)
                    for (int j = k; j < ns && j < k + nst; ++j)
                        mbar_wait_bounded(bar + j % nst, (uint32_t)((j / nst) & 1), DEFAULT_WAIT_CYCLES);
                __syncthreads();
                return;
            }
        }
        const float *sp = stage + (size_t)st * sb * V;
        if (k < nvs) {
            const int s0 = k * sb, s1 = min(nvr, s0 + sb);
#pragma unroll
            for (int p = 0; p < MAXP; ++p) {
                const int o = tid + p * blockDim.x;
                if (o >= npair) break;
                const int hl = o / V4, c4 = o - hl * V4;
                const int lo = hl * n, a0 = max(lo, s0), a1 = min(lo + n, s1);
                const float *w = wv + hl * W;
                for (int row = a0; row < a1; ++row)
                    fma4(acc[p], w[row - lo], lds4(sp + (size_t)(row - s0) * V + c4 * 4));
                if (lo + pos >= s0 && lo + pos < s1)  // append the step's value at slot pos
                    st4(A.vbuf + (((long long)b * H + h0 + hl) * W + pos) * V + c4 * 4,
                        lds4(sp + (size_t)(lo + pos - s0) * V + c4 * 4));
            }
        } else {
            const int s0 = (k - nvs) * sb, s1 = min(nbr, s0 + sb);
#pragma unroll
            for (int p = 0; p < MAXP; ++p) {
                const int o = tid + p * blockDim.x;
                if (o >= npair) break;
                const int hl = o / V4, c4 = o - hl * V4;
                const int qi = (h0 + hl) / hpq - q0;
                const float P = Ph[hl];
                const int r = m_rank[hl];
                const int lo = r > 0 ? m_rbs[hl] : RY + KDIM * m_didx[hl];
                const int a0 = max(lo, s0), a1 = min(lo + (r > 0 ? r : KDIM), s1);
                const float *cf = r > 0 ? dots + qi * dstride + W : qs + qi * KDIM;
                for (int row = a0; row < a1; ++row)
                    fma4(acc[p], P * cf[row - lo], lds4(sp + (size_t)(row - s0) * V + c4 * 4));
            }
        }
        __syncthreads();  // slot st consumed
        if (warp == 0 && k + nst < ns) {
            if (k + nst < nvs) issue_value(k + nst);
            else issue_base(k + nst);
        }
    }
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
        const int o = tid + p * blockDim.x;
        if (o >= npair) break;
        const int hl = o / V4, c4 = o - hl * V4;
        st4(A.y + ((long long)b * H + h0 + hl) * V + c4 * 4, acc[p]);
    }
}

// ring of stages: `nst` slots of `sb` rows
struct DgShape {
    int threads, maxp, nst, sb;
};

DgShape dg_shape(const DecodeArgs &a)
{
    DgShape s;
    const int pairs = a.Hg * (a.V / 4);
    s.threads = ((pairs + 31) / 32) * 32;
    if (s.threads < 128) s.threads = 128;
    if (s.threads > DG_MAX_THREADS) s.threads = DG_MAX_THREADS;
    const int need = (pairs + s.threads - 1) / s.threads;
    s.maxp = need <= 1 ? 1 : need <= 2 ? 2 : 4;  // at most 32 x 64 pairs over 512 threads
    s.nst = DG_STAGES;
    s.sb = DG_STAGE_BYTES / (4 * a.V);
    if (s.sb < 1) s.sb = 1;
    return s;
}

}  // namespace

bool decode_group_supported(const DecodeArgs &a)
{
    if (a.kind != SKETCHSSM_MAMBA2 || a.dense_all || a.Hg > MAX_HG) return false;
    const DgShape s = dg_shape(a);
    return dg_carve(a.V, a.W, a.Hg, a.Hg / a.hpq, a.cap, s.nst, s.sb).total <= 227 * 1024;
}

size_t decode_group_smem(const DecodeArgs &a)
{
    const DgShape s = dg_shape(a);
    return dg_carve(a.V, a.W, a.Hg, a.Hg / a.hpq, a.cap, s.nst, s.sb).total;
}

cudaError_t launch_decode_group(const DecodeArgs &a, cudaStream_t stream)
{
    if (a.B == 0) return cudaSuccess;
    const DgShape s = dg_shape(a);
    const size_t smem = dg_carve(a.V, a.W, a.Hg, a.Hg / a.hpq, a.cap, s.nst, s.sb).total;
    auto go = [&](auto kern) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<dim3((unsigned)((long long)a.B * a.G)), s.threads, smem, stream>>>(a, s.nst, s.sb);
        return cudaGetLastError();
    };
    switch (s.maxp) {
    case 1: return go(decode_group_kernel<1>);
    case 2: return go(decode_group_kernel<2>);
    default: return go(decode_group_kernel<4>);
    }
}

}  // namespace sk
