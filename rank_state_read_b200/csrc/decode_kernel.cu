// Sketch decode and dense-read decode: two launches per decode step.
//
// Paper abstract (SketchSSM, newx.sg / mlsanity pages): a decode step rebuilds the
// output from the sketch rows weighted by coefficients computed from the query, and
// never reads the full state; the keys and values buffered since the last state
// update (ReplaySSM) are replayed exactly.  A head with a dense fallback (PyPI page,
// stage "allocate") reads the full state instead; the dense-read baseline does that
// for every head.
//
// Every head's output is a weighted sum of rows of V floats: its base rows (the r
// sketch rows of Y, or the K state rows of S for a dense head) and its n buffered
// value rows.  The step splits into
//
//  1. the query-side products, written to the plan's scratch:
//     Mamba-2 (dots_kernel_mamba2), one CTA per (q/k head, 4 batch rows): the
//       group's basis rows, the rows' queries and buffered keys are staged in shared
//       memory by one round of cp.async; every product s_i = k_i . q and
//       u_m = Omega_g[m] . q is then one thread's loop over 128 staged floats, written
//       per (batch row, q/k head).  The step's key is appended to buffer slot pos.
//     GDN/KDA (coef_kernel_delta), one warp per (batch row, head): walk the buffer
//       newest first, x <- M_i^T x, keys (and KDA decays) prefetched four steps
//       ahead; the replay coefficients beta_i (k_i . x) and the base coefficients
//       Omega_g[m] . q0 (sketch) or q0 = x (dense) are written per head.  The step's
//       key, decay and beta are appended to buffer slot pos.
//  2. combine_kernel, one CTA per (work item, batch row): the layout kernel packs
//     the sketch heads of a basis group into items whose rows fit one shared-memory
//     stage (a dense head is an item of its own).  Warp 0 issues bulk (TMA) copies of
//     the item's block of Y (or the head's state), every buffered value row, the
//     step's values and the products of step 1, all counted on one mbarrier (the
//     item's record from the layout kernel is the only load on the path to the
//     copies; it is launched as a programmatic dependent of step 1 and waits for it
//     only before copying step 1's products).  After a bounded wait, thread (head,
//     column chunk) sums its head's
//     rows in row order (deterministic) and writes y.  For Mamba-2 the coefficients
//     are formed on the fly: walking the buffer newest first with w = 1,
//     row i gets w s_i and w <- w a_i, so that w ends as decay_prod; base row m then
//     gets decay_prod u_m (sketch) or decay_prod q_m (dense).  The step's value (and
//     Mamba-2's decay) is appended to buffer slot pos.
#include "device_util.cuh"
#include "internal.cuh"
#include "ptx_util.cuh"

namespace sk {
namespace {

constexpr int COMBINE_TARGET_THREADS = 160;
constexpr int STAGE_TARGET = 40 * 1024;  // bytes of rows of a typical sketch item
constexpr int MAXC = 32;
constexpr int COEF_THREADS = 128;

__host__ __device__ inline int round4(int x) { return (x + 3) & ~3; }

// Buffer position of batch row b: the call's pos, or the row's own (per-row positions).
// A position outside [0, W) is recorded (sketchssm_plan_check reports it) and -1 is
// returned: the caller then leaves the row alone.
__device__ __forceinline__ int row_position(const DecodeArgs &A, int b)
{
    if (!A.row_pos) return A.pos;
    const int p = __ldg(A.row_pos + b);
    if (p < 0 || p >= A.W) {
        atomicOr(A.status, SK_STATUS_BAD_ROW);
        return -1;
    }
    return p;
}

// ============================================================================ query-side products

constexpr int CM_THREADS = 256;
constexpr int CM_MINROWS = 4;   // batch rows per products CTA, at least
constexpr int CM_MAXROWS = 16;  // and at most
constexpr int OPAD = KDIM + 4;  // padded row: threads reading different rows hit different banks

struct CmCarve {
    size_t om, qs, ks, total;
    int kblock;  // floats per batch row of staged keys (W padded rows + 4: rows of different
                 // batch rows start 4 banks apart)
};

__host__ __device__ inline size_t cm_take(size_t &o, size_t bytes)
{
    const size_t r = o;
    o = (o + bytes + 127) & ~size_t(127);
    return r;
}

__host__ __device__ inline CmCarve cm_carve(int cap, int W, int rows)
{
    CmCarve c;
    c.kblock = W * OPAD + 4;
    size_t o = 0;
    c.om = cm_take(o, sizeof(float) * (size_t)cap * OPAD);
    c.qs = cm_take(o, sizeof(float) * (size_t)rows * OPAD);
    c.ks = cm_take(o, sizeof(float) * (size_t)rows * c.kblock);
    c.total = o;
    return c;
}

// Mamba-2: one CTA per (q/k head, `rows` batch rows).  Output per (batch row, q/k
// head): dots_row floats, s_0 .. s_{W-1} then u_0 .. u_{cap-1} (unused entries 0).
// One round of cp.async stages the group's basis rows, the rows' queries and keys (the
// step's key in slot pos); then every dot product s_i = k_i . q and u_m = Omega_g[m] . q
// is one thread's loop over 128 staged floats.  Task t = (row t / rows, batch row
// t % rows): the threads of a quarter-warp read one basis row (broadcast) or keys and
// queries of different batch rows (padded to fall on different banks).  The step's key
// is appended to buffer slot pos.
__global__ void __launch_bounds__(CM_THREADS)
dots_kernel_mamba2(const DecodeArgs A)
{
    extern __shared__ __align__(128) unsigned char cms[];
    pdl_launch_dependents();  // the combine may start staging its rows now
    const int tid = threadIdx.x;
    const int W = A.W, hpq = A.hpq, cap = A.cap, dr = A.dots_row;
    const int rows = A.cm_rows;
    const int q = blockIdx.x, b0 = blockIdx.y * rows;
    const int nb = min(rows, A.B - b0);
    // buffer position of each of the CTA's rows (-1: a bad per-row position, row
    // skipped); all rows at the call's pos unless the call gives per-row positions
    __shared__ int rpos_s[CM_MAXROWS];
    int nmax = A.pos + 1;  // key slots in use in any of the rows
    if (A.row_pos) {
        if (tid < nb) rpos_s[tid] = row_position(A, b0 + tid);
        __syncthreads();
        nmax = 0;
        for (int bl = 0; bl < nb; ++bl) nmax = max(nmax, rpos_s[bl] + 1);
    }
    auto rpos = [&](int bl) { return A.row_pos ? rpos_s[bl] : A.pos; };
    const int g = (q * hpq) / A.Hg;
    const CmCarve cv = cm_carve(cap, W, rows);
    float *om = reinterpret_cast<float *>(cms + cv.om);  // [rq][OPAD]
    float *qs = reinterpret_cast<float *>(cms + cv.qs);  // [rows][OPAD]
    float *ks = reinterpret_cast<float *>(cms + cv.ks);  // [rows][kblock]: key i at i OPAD

    const int rq = A.dense_all ? 0 : __ldg(A.qk_rneed + q);
    const float *og = A.omega + (long long)g * A.Rb * KDIM;
    for (int x = tid; x < rq * (KDIM / 4); x += CM_THREADS) {
        const int j = x >> 5, c = x & 31;
        cp_async16(om + j * OPAD + c * 4, og + (long long)j * KDIM + c * 4);
    }
    for (int x = tid; x < nb * (KDIM / 4); x += CM_THREADS) {
        const int bl = x >> 5, c = x & 31;
        cp_async16(qs + bl * OPAD + c * 4, A.q + ((long long)(b0 + bl) * A.Hqk + q) * KDIM + c * 4);
    }
    for (int x = tid; x < nb * nmax * (KDIM / 4); x += CM_THREADS) {
        const int c = x & 31, r = x >> 5, bl = r / nmax, i = r - bl * nmax, pos = rpos(bl);
        if (i > pos) continue;
        const long long qrow = (long long)(b0 + bl) * A.Hqk + q;
        cp_async16(ks + bl * cv.kblock + i * OPAD + c * 4,
                   (i == pos ? A.k + qrow * KDIM : A.kbuf + (qrow * W + i) * KDIM) + c * 4);
    }
    cp_async_commit();
    // unused entries of the rows: 0
    for (int x = tid; x < nb * dr; x += CM_THREADS) {
        const int bl = x / dr, e = x - bl * dr;
        if (rpos(bl) < 0) continue;
        if ((e > rpos(bl) && e < W) || e >= W + rq) A.scratch[((long long)(b0 + bl) * A.Hqk + q) * dr + e] = 0.f;
    }
    cp_async_wait<0>();
    __syncthreads();

    // task (row rr, batch row): rr < nmax a key slot, else basis row rr - nmax
    for (int t = tid; t < (nmax + rq) * nb; t += CM_THREADS) {
        const int rr = t / nb, bl = t - rr * nb;
        if (rr < nmax && rr > rpos(bl)) continue;
        const float *row = rr < nmax ? ks + bl * cv.kblock + rr * OPAD : om + (size_t)(rr - nmax) * OPAD;
        const float *qb = qs + (size_t)bl * OPAD;
        float4 acc = zero4();
#pragma unroll 8
        for (int c = 0; c < KDIM; c += 4) {
            const float4 o = lds4(row + c), v = lds4(qb + c);
            acc.x = fmaf(o.x, v.x, acc.x);
            acc.y = fmaf(o.y, v.y, acc.y);
            acc.z = fmaf(o.z, v.z, acc.z);
            acc.w = fmaf(o.w, v.w, acc.w);
        }
        A.scratch[((long long)(b0 + bl) * A.Hqk + q) * dr + (rr < nmax ? rr : W + rr - nmax)] =
            (acc.x + acc.y) + (acc.z + acc.w);
    }
    // the step's key goes to buffer slot pos (from the stage)
    for (int x = tid; x < nb * (KDIM / 4); x += CM_THREADS) {
        const int bl = x >> 5, c = x & 31, pos = rpos(bl);
        if (pos < 0) continue;
        const long long qrow = (long long)(b0 + bl) * A.Hqk + q;
        st4(A.kbuf + (qrow * W + pos) * KDIM + c * 4, lds4(ks + bl * cv.kblock + pos * OPAD + c * 4));
    }
}

// GDN / KDA: one warp per (head, batch row).
template <int KIND>
__global__ void __launch_bounds__(COEF_THREADS)
coef_kernel_delta(const DecodeArgs A)
{
    pdl_launch_dependents();  // the combine may start staging its rows now
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h = blockIdx.x * (COEF_THREADS / 32) + warp, b = blockIdx.y;
    if (h >= A.H) return;
    const int pos = row_position(A, b);
    if (pos < 0) return;
    const int H = A.H, W = A.W, n = pos + 1, hpq = A.hpq;
    const int qk = h / hpq, g = h / A.Hg;
    const long long bh = (long long)b * H + h;
    const long long qrow = (long long)b * A.Hqk + qk;
    const int r = __ldg(A.rank + h);
    const bool dense = A.dense_all || r <= 0;
    const int rb = dense ? KDIM : r;
    float *dst = A.scratch + (long long)b * A.coef_row +
                 (A.dense_all ? (long long)h * A.coef_dense_block : __ldg(A.coff + h));

    float bl = 0.f, al = 0.f;
    if (lane < n) {
        bl = (lane == pos) ? __ldg(A.beta + bh) : __ldg(A.bbuf + bh * W + lane);
        if (KIND == SKETCHSSM_GDN) al = (lane == pos) ? __ldg(A.a + bh) : __ldg(A.abuf + bh * W + lane);
    }
    if (lane == pos) {
        A.bbuf[bh * W + pos] = bl;
        if (KIND == SKETCHSSM_GDN) A.abuf[bh * W + pos] = al;
    }
    const float *kcur = A.k + qrow * KDIM + lane * 4;
    const float *kb = A.kbuf + qrow * W * KDIM + lane * 4;
    const float *acur = A.a + bh * KDIM + lane * 4;      // KDA
    const float *ab = A.abuf + bh * W * KDIM + lane * 4;  // KDA
    auto kl = [&](int i) { return i == pos ? ldg4(kcur) : ldg4(kb + (long long)i * KDIM); };
    auto al4 = [&](int i) { return i == pos ? ldg4(acur) : ldg4(ab + (long long)i * KDIM); };
    const float4 z = zero4();
    float4 k0 = kl(n - 1), k1 = n >= 2 ? kl(n - 2) : z, k2 = n >= 3 ? kl(n - 3) : z, k3 = n >= 4 ? kl(n - 4) : z;
    float4 a0 = z, a1 = z, a2 = z, a3 = z;
    if (KIND == SKETCHSSM_KDA) {
        a0 = al4(n - 1);
        if (n >= 2) a1 = al4(n - 2);
        if (n >= 3) a2 = al4(n - 3);
        if (n >= 4) a3 = al4(n - 4);
    }
    float4 x = ldg4(A.q + qrow * KDIM + lane * 4);
    for (int i = n - 1; i >= 0; --i) {
        const float4 kv = k0;
        k0 = k1;
        k1 = k2;
        k2 = k3;
        k3 = (i >= 4) ? kl(i - 4) : z;
        float4 av = z;
        if (KIND == SKETCHSSM_KDA) {
            av = a0;
            a0 = a1;
            a1 = a2;
            a2 = a3;
            a3 = (i >= 4) ? al4(i - 4) : z;
        }
        const float bi = __shfl_sync(0xffffffffu, bl, i);
        const float s1 = warp_sum(dot4(kv, x));
        if (lane == 0) dst[rb + i] = bi * s1;
        if (KIND == SKETCHSSM_GDN) {
            const float ai = __shfl_sync(0xffffffffu, al, i);
            const float t = bi * s1;
            x.x = ai * fmaf(-t, kv.x, x.x);
            x.y = ai * fmaf(-t, kv.y, x.y);
            x.z = ai * fmaf(-t, kv.z, x.z);
            x.w = ai * fmaf(-t, kv.w, x.w);
        } else {
            const float4 xa = make_float4(av.x * x.x, av.y * x.y, av.z * x.z, av.w * x.w);
            const float t = bi * warp_sum(dot4(kv, xa));
            x.x = fmaf(-t, kv.x, xa.x);
            x.y = fmaf(-t, kv.y, xa.y);
            x.z = fmaf(-t, kv.z, xa.z);
            x.w = fmaf(-t, kv.w, xa.w);
        }
        if (i == pos) {
            if (h == qk * hpq) st4(A.kbuf + (qrow * W + pos) * KDIM + lane * 4, kv);
            if (KIND == SKETCHSSM_KDA) st4(A.abuf + (bh * W + pos) * KDIM + lane * 4, av);
        }
    }
    // x = q0: base coefficients
    if (dense) {
        st4(dst + lane * 4, x);
    } else {
        const float *og = A.omega + (long long)g * A.Rb * KDIM + lane * 4;
        for (int j0 = 0; j0 < rb; j0 += 8) {
            float4 om[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) om[u] = (j0 + u < rb) ? ldg4(og + (long long)(j0 + u) * KDIM) : z;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (j0 + u >= rb) break;
                const float d = warp_sum(dot4(om[u], x));
                if (lane == 0) dst[j0 + u] = d;
            }
        }
    }
}

// ============================================================================ combine

struct Carve {
    size_t bar, meta, coef, dots, qrow, as, stage, total;
};

__host__ __device__ inline size_t take(size_t &o, size_t bytes)
{
    const size_t r = o;
    o = (o + bytes + 127) & ~size_t(127);
    return r;
}

__host__ __device__ inline Carve carve(int kind, int stage_rows, int coef_cap, int V, int W, int maxnh,
                                       int dots_row)
{
    const bool m2 = kind == SKETCHSSM_MAMBA2;
    Carve c;
    size_t o = 0;
    c.bar = take(o, 16);
    c.meta = take(o, sizeof(int) * (6 * MAXC + 8));
    c.coef = take(o, m2 ? 0 : sizeof(float) * (size_t)coef_cap);
    c.dots = take(o, m2 ? sizeof(float) * (size_t)maxnh * dots_row : 0);
    c.qrow = take(o, m2 ? sizeof(float) * KDIM : 0);
    c.as = take(o, m2 ? sizeof(float) * (size_t)maxnh * W : 0);
    c.stage = take(o, sizeof(float) * (size_t)stage_rows * V);
    c.total = o;
    return c;
}

template <int KIND>
__global__ void __launch_bounds__(256)
combine_kernel(const DecodeArgs A)
{
    constexpr bool M2 = KIND == SKETCHSSM_MAMBA2;
    extern __shared__ __align__(128) unsigned char smem[];
    const Carve cv = carve(KIND, A.stage_rows, A.coef_cap, A.V, A.W, A.maxnh, A.dots_row);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + cv.bar);
    int *meta = reinterpret_cast<int *>(smem + cv.meta);
    int *hs = meta, *rb = meta + MAXC, *rbs = meta + 2 * MAXC, *cc = meta + 3 * MAXC, *ch = meta + 4 * MAXC;
    float *coef = reinterpret_cast<float *>(smem + cv.coef);
    float *dots = reinterpret_cast<float *>(smem + cv.dots);
    float *qrow_s = reinterpret_cast<float *>(smem + cv.qrow);
    float *as_s = reinterpret_cast<float *>(smem + cv.as);
    float *stage = reinterpret_cast<float *>(smem + cv.stage);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.y;
    const int pos = row_position(A, b);
    if (pos < 0) return;
    const int H = A.H, V = A.V, W = A.W, n = pos + 1, hpq = A.hpq, dr = A.dots_row;
    // per-row positions: this row's work list (the launch covers the longest list)
    const int *rec_list = A.rec;
    if (A.row_pos && !A.dense_all) {
        if ((int)blockIdx.x >= __ldg(A.counts + 2 + n)) return;
        rec_list = A.rec + (size_t)(n - 1) * (H + A.G) * 8;
    }
    // the item's record: {entry, span, member mask, rows R, off[h_first], coff[h_first], coef floats, h_first}
    int R, yrow0, c0, cfl, h_first, span;
    unsigned mask;
    bool dense;
    if (A.dense_all) {
        dense = true;
        h_first = blockIdx.x;
        span = 1;
        mask = 1u;
        R = KDIM;
        yrow0 = 0;
        c0 = h_first * A.coef_dense_block;
        cfl = A.coef_dense_block;
    } else {
        const int4 r0 = __ldg(reinterpret_cast<const int4 *>(rec_list) + 2 * blockIdx.x);
        const int4 r1 = __ldg(reinterpret_cast<const int4 *>(rec_list) + 2 * blockIdx.x + 1);
        dense = r0.x < 0;
        span = r0.y;
        mask = (unsigned)r0.z;
        R = r0.w;
        yrow0 = r1.x;
        c0 = r1.y;
        cfl = r1.z;
        h_first = r1.w;
    }
    const int nh = __popc(mask);

    if (warp == 0) {
        const int h = h_first + lane;
        const bool member = (mask >> lane) & 1u;
        const unsigned below = mask & ((1u << lane) - 1u);
        const int slot = __popc(below);
        // Mamba-2: the q/k heads (chains) of the members, in order
        const int qk = h / hpq;
        const int qk_prev = __shfl_sync(0xffffffffu, qk, below ? 31 - __clz(below) : lane);
        const bool new_chain = M2 && member && (slot == 0 || qk != qk_prev);
        const unsigned cmask = __ballot_sync(0xffffffffu, new_chain);
        const int chain = __popc(cmask & ((2u << lane) - 1u)) - 1;
        const int nch = __popc(cmask);
        if (lane == 0) {
            mbar_init(bar, 1);
            mbar_fence_init();
            uint32_t bytes = (uint32_t)((R + nh * n) * V * 4);
            bytes += M2 ? (uint32_t)(nch * dr * 4 + (dense ? KDIM * 4 : 0)) : (uint32_t)(cfl * 4);
            mbar_arrive_expect_tx(bar, bytes);
            const float *src = dense ? A.S + ((long long)b * H + h_first) * KDIM * V
                                     : A.Y + ((long long)b * A.rtot + yrow0) * V;
            bulk_copy_g2s(stage, src, (uint32_t)(R * V * 4), bar);
            if (M2 && dense) bulk_copy_g2s(qrow_s, A.q + ((long long)b * A.Hqk + qk) * KDIM, KDIM * 4, bar);
        }
        __syncwarp();
        // stage rows: [item's Y block or state: R][member slot's buffered values: pos each]
        // [the step's values: one per member]; when the members are a contiguous run of
        // heads their step values are one contiguous run of v, so one copy brings them all
        const long long bh = (long long)b * H + h;
        if (member) {
            if (pos > 0)
                bulk_copy_g2s(stage + (size_t)(R + slot * pos) * V, A.vbuf + bh * W * V, (uint32_t)(pos * V * 4), bar);
            if (span != nh) bulk_copy_g2s(stage + (size_t)(R + nh * pos + slot) * V, A.v + bh * V, (uint32_t)(V * 4), bar);
        }
        if (span == nh && lane == 0)
            bulk_copy_g2s(stage + (size_t)(R + nh * pos) * V, A.v + ((long long)b * H + h_first) * V,
                          (uint32_t)(nh * V * 4), bar);
        // the products of the first launch of this step: wait until it has finished
        pdl_wait_primary();
        if (!M2 && lane == 0)
            bulk_copy_g2s(coef, A.scratch + (long long)b * A.coef_row + c0, (uint32_t)(cfl * 4), bar);
        if (new_chain)
            bulk_copy_g2s(dots + (size_t)chain * dr, A.scratch + ((long long)b * A.Hqk + qk) * dr,
                          (uint32_t)(dr * 4), bar);
        // per-member layout (off the copies' path)
        const int rbv = member ? (dense ? KDIM : __ldg(A.rank + h)) : 0;
        int incl = rbv, cinc = member ? round4(rbv + W) : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            const int u = __shfl_up_sync(0xffffffffu, cinc, o);
            if (lane >= o) {
                incl += t;
                cinc += u;
            }
        }
        if (member) {
            hs[slot] = h;
            rb[slot] = rbv;
            rbs[slot] = incl - rbv;
            cc[slot] = cinc - round4(rbv + W);
            ch[slot] = chain;
        }
    }
    if (M2) {
        // decays of the members' buffered tokens, spread over the CTA (one round of
        // loads, in flight with the bulk copies); the step's decay goes to slot pos
        for (int x = tid; x < nh * n; x += blockDim.x) {
            const int slot = x / n, i = x - slot * n;
            const long long bh = (long long)b * H + h_first + (int)__fns(mask, 0, slot + 1);
            const float av = (i == pos) ? __ldg(A.a + bh) : __ldg(A.abuf + bh * W + i);
            as_s[slot * W + i] = av;
            if (i == pos) A.abuf[bh * W + pos] = av;
        }
    }
    __syncthreads();
    // a wait past the plan's limit is recorded (sketchssm_plan_check reports it) and then
    // continued up to DEFAULT_WAIT_CYCLES; only a wait that outlasts both gives up
    bool ok = mbar_wait_bounded(bar, 0, A.wait_limit);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) atomicOr(A.status, SK_STATUS_DECODE_TIMEOUT);
        ok = mbar_wait_bounded(bar, 0, DEFAULT_WAIT_CYCLES);
        if (__syncthreads_or(!ok)) {
            // give up: let the copies still in flight land (bounded) before the CTA exits
            if (tid == 0) mbar_wait_bounded(bar, 0, DEFAULT_WAIT_CYCLES);
            __syncthreads();
            return;
        }
    }
    const int V4 = V >> 2;
    for (int o = tid; o < nh * V4; o += blockDim.x) {
        const int hl = o / V4, c4 = o - hl * V4;
        const int r0 = rbs[hl], rbh = rb[hl];
        const int rv = R + hl * pos, rcur = R + nh * pos + hl;  // buffered values, the step's value
        const float *sp = stage + c4 * 4;
        float4 acc0 = zero4(), acc1 = zero4();
        if (M2) {
            const float *sv = dots + (size_t)ch[hl] * dr;
            const float *uv = dense ? qrow_s : sv + W;
            const float *av = as_s + hl * W;
            // prod_{j>i} a_j, newest token first; ends as decay_prod
            fma4(acc1, sv[pos], lds4(sp + (size_t)rcur * V));
            float w = av[pos];
            for (int i = pos - 1; i >= 0; --i) {
                fma4(acc1, w * sv[i], lds4(sp + (size_t)(rv + i) * V));
                w *= av[i];
            }
            int j = 0;
            for (; j + 1 < rbh; j += 2) {
                fma4(acc0, w * uv[j], lds4(sp + (size_t)(r0 + j) * V));
                fma4(acc1, w * uv[j + 1], lds4(sp + (size_t)(r0 + j + 1) * V));
            }
            if (j < rbh) fma4(acc0, w * uv[j], lds4(sp + (size_t)(r0 + j) * V));
        } else {
            const float *cf = coef + cc[hl];
            int j = 0;
            for (; j + 1 < rbh; j += 2) {
                fma4(acc0, cf[j], lds4(sp + (size_t)(r0 + j) * V));
                fma4(acc1, cf[j + 1], lds4(sp + (size_t)(r0 + j + 1) * V));
            }
            if (j < rbh) fma4(acc0, cf[j], lds4(sp + (size_t)(r0 + j) * V));
            for (int i = 0; i < pos; ++i) fma4(acc1, cf[rbh + i], lds4(sp + (size_t)(rv + i) * V));
            fma4(acc1, cf[rbh + pos], lds4(sp + (size_t)rcur * V));
        }
        const float4 acc = make_float4(acc0.x + acc1.x, acc0.y + acc1.y, acc0.z + acc1.z, acc0.w + acc1.w);
        const long long bh = (long long)b * H + hs[hl];
        st4(A.y + bh * V + c4 * 4, acc);
        st4(A.vbuf + (bh * W + pos) * V + c4 * 4, lds4(sp + (size_t)rcur * V));
    }
}

template <int KIND>
cudaError_t launch_combine(const DecodeArgs &a, cudaStream_t stream)
{
    const size_t smem = decode_smem_bytes(a);
    cudaError_t e = cudaFuncSetAttribute(combine_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: CTAs may start while the products kernel runs
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.n_items, a.B);
    cfg.blockDim = dim3(a.threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, combine_kernel<KIND>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

int dots_row(int W, int cap) { return round4(W + cap); }

bool decode_geometry(int kind, int V, int W, int cap, int Hg, DecodeGeometry *gm)
{
    const int V4 = V / 4;
    // items may hold a whole group: the row budget bounds their bytes, and the row sums
    // loop over (head, column chunk) outputs when they outnumber the threads
    const int m = Hg < MAXC ? Hg : MAXC;
    gm->maxnh = m;
    int per = COMBINE_TARGET_THREADS / V4;
    if (per < 1) per = 1;
    if (per > m) per = m;
    int t = ((per * V4 + 31) / 32) * 32;
    if (t < 64) t = 64;
    if (t > 256) t = 256;
    gm->threads = t;
    int rows = STAGE_TARGET / (4 * V);
    if (rows < KDIM + W) rows = KDIM + W;
    if (rows < cap + W) rows = cap + W;
    gm->stage_rows = rows;
    gm->coef_cap = rows + m * (W + 3) + 4;
    return carve(kind, rows, gm->coef_cap, V, W, m, dots_row(W, cap)).total <= 227 * 1024 &&
           cm_carve(cap, W, 1).total <= 227 * 1024;
}

int coef_block(int rows, int W) { return round4(rows + W); }

int coef_rows(int cap, int W, int B, int Hqk, int sms)
{
    // the fewest batch rows per CTA (at least CM_MINROWS) whose grid of Hqk x B / rows
    // CTAs runs in one wave at the occupancy its shared memory allows: a partial second
    // wave would cost a whole CTA lifetime of this latency-bound kernel
    for (int rows = CM_MINROWS; rows <= CM_MAXROWS; ++rows) {
        const size_t smem = cm_carve(cap, W, rows).total;
        int per_sm = (int)((227 * 1024) / (smem + 1024));
        if (per_sm > 2048 / CM_THREADS) per_sm = 2048 / CM_THREADS;
        if (per_sm < 1) break;
        const long long ctas = (long long)Hqk * ((B + rows - 1) / rows);
        if (ctas <= (long long)sms * per_sm) return rows;
    }
    return CM_MINROWS;
}

size_t decode_smem_bytes(const DecodeArgs &a)
{
    return carve(a.kind, a.stage_rows, a.coef_cap, a.V, a.W, a.maxnh, a.dots_row).total;
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream)
{
    if (a.B == 0) return cudaSuccess;
    cudaError_t e;
    if (a.kind == SKETCHSSM_MAMBA2) {
        const size_t cm = cm_carve(a.cap, a.W, a.cm_rows).total;
        if ((e = cudaFuncSetAttribute(dots_kernel_mamba2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cm)) !=
            cudaSuccess)
            return e;
        dots_kernel_mamba2<<<dim3(a.Hqk, (a.B + a.cm_rows - 1) / a.cm_rows), CM_THREADS, cm, stream>>>(a);
    } else {
        const dim3 grid((a.H + COEF_THREADS / 32 - 1) / (COEF_THREADS / 32), a.B);
        if (a.kind == SKETCHSSM_GDN) coef_kernel_delta<SKETCHSSM_GDN><<<grid, COEF_THREADS, 0, stream>>>(a);
        else coef_kernel_delta<SKETCHSSM_KDA><<<grid, COEF_THREADS, 0, stream>>>(a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (a.n_items == 0) return cudaSuccess;
    switch (a.kind) {
    case SKETCHSSM_MAMBA2: return launch_combine<SKETCHSSM_MAMBA2>(a, stream);
    case SKETCHSSM_GDN: return launch_combine<SKETCHSSM_GDN>(a, stream);
    default: return launch_combine<SKETCHSSM_KDA>(a, stream);
    }
}

}  // namespace sk
