// Flush: the write-full step (one launch every W decode steps).
//
// SketchSSM (paper abstract): the state keeps receiving every update in full, and
// the only time it is read is at a state update, where one pass over it computes the
// outputs for the fixed basis vectors and stores them as the compact sketch.  For
// every (batch row, head):
//   1. apply the n buffered tokens in order, S <- M_i S + beta_i k_i v_i^T
//      (Mamba-2 in closed form: S <- P S + sum_i w_i k_i v_i^T with
//       P = prod_i a_i, w_i = prod_{j>i} a_j);
//   2. write S back (skipped when n = 0);
//   3. for a sketch head, Y[off + m] = Omega_g[m] S for m < rank, from the S still
//      held in registers, so S crosses HBM once each way.
//
// Work item: (b, h, column slab of VS columns); columns of S evolve independently,
// so a slab is self-contained.  A persistent CTA walks a contiguous range of items
// (consecutive heads of a batch row) with VS/16 compute warps and one producer warp.
// Each compute warp owns 16 columns of the slab and holds them for all 128 state rows
// in registers (64 fp32 a thread).
//   Mamba-2: the rank-n update S <- P S + K^T (w o V) runs on the tensor cores
//   (mma.sync m16n8k8, tf32 operands split as x = hi + lo with the three products
//   hi hi + hi lo + lo hi, which keeps fp32 accuracy); the state lives in the
//   accumulator layout (columns 8 nt + 2 t (+1) for lane 4 g + t, and a fixed map of
//   accumulator rows to state rows that keeps the fragment reads of the padded 4-row
//   chunks conflict-free).  Staged value rows carry 8 floats of padding, key rows 4.
//   GDN / KDA: thread (ks, c4) holds the float4 column chunk c4 of the 16 state rows
//   4 ks + 32 q + e (q, e < 4) and applies the delta rule token by token; every
//   reduction over k stays inside the warp, and the float4 reads of keys and decays by
//   the 8 row slices are 128 consecutive bytes.
// Both then project the new state onto the basis rows on the FP32 pipe and write S and
// the sketch rows straight from registers.
//
// Data movement is TMA bulk copies (cp.async.bulk, completion counted on an mbarrier),
// which keep far more bytes in flight per SM than register loads.  The producer warp
// requests, one item ahead:
//   - the item's state slab into one shared buffer, as 32 chunks of 4 rows, each
//     chunk padded by 4 floats (so that the reads of all threads of a warp fall on
//     disjoint banks);
//   - the buffered keys, values and KDA decays into one of two token buffers;
//   - when the head group changes, the basis rows 0 .. rmax_g - 1 of the new group,
//     which stay resident while the group lasts.
// Handshake: `full` completes when an item's copies have landed; every compute warp
// arrives on `empty` once it has the slab in registers (by then it is also done with
// the previous item), which frees the slab buffer, the other token buffer and the
// basis rows for the producer.  No CTA-wide barrier in the loop.  State and sketch rows
// are written straight from registers; the per-token scalars a_i, beta_i are loaded
// one item ahead into the lanes < n and broadcast by shuffles.
#include "device_util.cuh"
#include "internal.cuh"
#include "ptx_util.cuh"

namespace sk {
namespace {

constexpr int QROWS = KDIM / 32;  // row quads per thread (4): rows 4 ks + 32 q + e
constexpr int FLUSH_MAXT = 192;   // up to 5 compute warps (VS <= 80) + the producer

struct FlushCarve {
    size_t bar, S, T, O, AF, total;      // byte offsets in shared memory
    size_t tkeys, tv, ta, tfloats;       // float offsets within one token buffer
    int ks, vs;                          // row strides (floats) of staged keys and values
};

// Mamba-2 token rows are staged padded: values by 8 floats (the B-fragment reads of 4
// tokens x 8 columns hit 32 distinct banks), keys by 4 (the A-fragment reads of 4 tokens
// x 8 state rows spaced 8 apart hit 8 banks, 4 lanes each)
constexpr int MPAD_V = 8, MPAD_K = 4;

__host__ __device__ inline size_t align128(size_t x) { return (x + 127) & ~size_t(127); }

__host__ __device__ inline FlushCarve flush_carve(int kind, int VS, int W, int rcap)
{
    FlushCarve c;
    const bool m2 = kind == SKETCHSSM_MAMBA2;
    c.ks = m2 ? KDIM + MPAD_K : KDIM;
    c.vs = m2 ? VS + MPAD_V : VS;
    c.tkeys = 0;
    c.tv = (size_t)W * c.ks;
    c.ta = c.tv + (size_t)W * c.vs;
    c.tfloats = c.ta + (kind == SKETCHSSM_KDA ? (size_t)W * KDIM : 0);
    size_t o = 0;
    c.bar = o;  // full, empty, omega barriers and the abort flag
    o = align128(o + 4 * sizeof(uint64_t));
    c.S = o;
    o = align128(o + sizeof(float) * 32 * (size_t)(4 * VS + 4));
    c.T = o;
    o = align128(o + 2 * sizeof(float) * c.tfloats);
    c.O = o;
    o = align128(o + sizeof(float) * (size_t)rcap * KDIM);
    c.AF = o;  // Mamba-2: split key fragments, [k-step][m-tile][hi, lo][lane][4]
    o = align128(o + (m2 ? sizeof(float) * (size_t)((W + 7) / 8) * 8 * 32 * 8 : 0));
    c.total = o;
    return c;
}

// Tokens a batch row applies: the call's n, or the row's own count (per-row counts).
// A count outside [0, W] is recorded (sketchssm_plan_check reports it) and the row is
// left alone (0).
__device__ __forceinline__ int row_tokens(const FlushArgs &A, int b)
{
    if (!A.row_n) return A.n;
    const int n = __ldg(A.row_n + b);
    if (n < 0 || n > A.W) {
        atomicOr(A.status, SK_STATUS_BAD_ROW);
        return 0;
    }
    return n;
}

// (b, h, slab) of consecutive items, advanced without divisions; the head's rank and
// sketch-row offset are loaded when the cursor moves (one item before they are used).
// n: the row's tokens; proj: whether the item re-forms its sketch rows (a sketch head,
// and with per-row counts only a row that applies tokens)
struct Cursor {
    int b, h, slab, r, off, n;
    bool proj;
    __device__ void init(const FlushArgs &A, long long item, int nslab)
    {
        const long long bh = item / nslab;
        slab = (int)(item - bh * nslab);
        b = (int)(bh / A.H);
        h = (int)(bh - (long long)b * A.H);
        r = __ldg(A.rank + h);
        off = __ldg(A.off + h);
        n = row_tokens(A, b);
        proj = r > 0 && (!A.row_n || n > 0);
    }
    __device__ void next(const FlushArgs &A, int nslab)
    {
        if (++slab == nslab) {
            slab = 0;
            if (++h == A.H) {
                h = 0;
                ++b;
                n = row_tokens(A, b);
            }
            r = __ldg(A.rank + h);
            off = __ldg(A.off + h);
            proj = r > 0 && (!A.row_n || n > 0);
        }
    }
    __device__ long long bh(const FlushArgs &A) const { return (long long)b * A.H + h; }
};

// Wait for phase `parity` of `bar`, giving up after `limit` cycles or when another
// warp of the CTA has given up (abort flag set).
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, long long limit,
                                              const volatile int *abort)
{
    const long long t0 = clock64();
    while (!mbar_poll(bar, parity, limit)) {
        if (*abort || clock64() - t0 > limit) return false;
    }
    return true;
}

// A wait past the plan's limit is recorded in the plan's status word (a timeout that
// sketchssm_plan_check reports) and then continued, up to DEFAULT_WAIT_CYCLES more, for
// the same phase, so that the copy protocol stays in order.  Only a wait that outlasts
// both gives up: it sets the CTA's abort flag and returns false.
__device__ __forceinline__ bool staged_wait(uint64_t *bar, uint32_t parity, const FlushArgs &A,
                                            volatile int *abort)
{
    if (wait_or_abort(bar, parity, A.wait_limit, abort)) return true;
    if (*abort) return false;
    atomicOr(A.status, SK_STATUS_FLUSH_TIMEOUT);
    if (wait_or_abort(bar, parity, DEFAULT_WAIT_CYCLES, abort)) return true;
    *abort = 1;
    return false;
}

// The producer warp requests an item's state slab and (n > 0) its buffered tokens,
// all counted on `bar`.  An item with nothing to do (n = 0 and a dense head) arrives
// on the barrier with no bytes.
template <int KIND>
__device__ __forceinline__ void issue_item(const FlushArgs &A, const Cursor &it, int nslab, float *Sbuf,
                                           float *T, const FlushCarve &cv, uint64_t *bar, int lane, bool keys)
{
    const int V = A.V, VS = A.VS, W = A.W, n = it.n;
    const bool needed = n > 0 || it.proj;
    if (KIND != SKETCHSSM_MAMBA2) keys = true;
    if (lane == 0) {
        uint32_t bytes = 0;
        if (needed) {
            bytes = (uint32_t)(KDIM * VS * 4);
            if (n > 0) {
                bytes += (uint32_t)((keys ? n * KDIM * 4 : 0) + n * VS * 4);
                if (KIND == SKETCHSSM_KDA) bytes += (uint32_t)(n * KDIM * 4);
            }
        }
        mbar_arrive_expect_tx(bar, bytes);
    }
    __syncwarp();
    if (!needed) return;
    const long long bh = it.bh(A);
    const float *Sg = A.S + bh * KDIM * V + (long long)it.slab * VS;
    float *dst = Sbuf + (size_t)lane * (4 * VS + 4);
    if (nslab == 1) {  // 4 state rows are 4 V contiguous floats
        bulk_copy_g2s(dst, Sg + (long long)lane * 4 * V, (uint32_t)(16 * VS), bar);
    } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
            bulk_copy_g2s(dst + e * VS, Sg + (long long)(lane * 4 + e) * V, (uint32_t)(4 * VS), bar);
    }
    if (KIND == SKETCHSSM_MAMBA2) {  // keys (only for a new key set) and values, one padded row each
        if (n > 0 && lane < n) {
            const int qk = it.h / A.hpq;
            if (keys)
                bulk_copy_g2s(T + cv.tkeys + (size_t)lane * cv.ks,
                              A.kbuf + (((long long)it.b * A.Hqk + qk) * W + lane) * KDIM, (uint32_t)(KDIM * 4), bar);
            bulk_copy_g2s(T + cv.tv + (size_t)lane * cv.vs, A.vbuf + (bh * W + lane) * V + (long long)it.slab * VS,
                          (uint32_t)(VS * 4), bar);
        }
        return;
    }
    if (n > 0) {
        const int qk = it.h / A.hpq;
        if (lane == 0)
            bulk_copy_g2s(T + cv.tkeys, A.kbuf + ((long long)it.b * A.Hqk + qk) * W * KDIM,
                          (uint32_t)(n * KDIM * 4), bar);
        if (KIND == SKETCHSSM_KDA && lane == 1)
            bulk_copy_g2s(T + cv.ta, A.abuf + bh * W * KDIM, (uint32_t)(n * KDIM * 4), bar);
        const float *vg = A.vbuf + bh * W * V + (long long)it.slab * VS;
        if (nslab == 1) {
            if (lane == 2) bulk_copy_g2s(T + cv.tv, vg, (uint32_t)(n * V * 4), bar);
        } else {
            for (int i = lane; i < n; i += 32)
                bulk_copy_g2s(T + cv.tv + (size_t)i * VS, vg + (long long)i * V, (uint32_t)(VS * 4), bar);
        }
    }
}

// acc += sum_e c_e s[e] over a row quad
__device__ __forceinline__ void quad_dot(float4 &acc, float4 c, const float4 *s)
{
    fma4(acc, c.x, s[0]);
    fma4(acc, c.y, s[1]);
    fma4(acc, c.z, s[2]);
    fma4(acc, c.w, s[3]);
}

__device__ __forceinline__ float4 add4(float4 a, float4 b)
{
    return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

__device__ __forceinline__ float4 shfl_xor4(float4 v, int m)
{
    return make_float4(__shfl_xor_sync(0xffffffffu, v.x, m), __shfl_xor_sync(0xffffffffu, v.y, m),
                       __shfl_xor_sync(0xffffffffu, v.z, m), __shfl_xor_sync(0xffffffffu, v.w, m));
}

// x = hi + lo with hi, lo tf32 (round to nearest, ties away): hi carries the top 11
// significant bits, lo the next 11, so hi hi + hi lo + lo hi misses only lo lo
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo)
{
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
    const float rest = x - __uint_as_float(hi);
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(rest));
}

// d += a b for one 16 x 8 x 8 tf32 tile (fp32 accumulate), fragments as in the PTX ISA
// (lane 4 g + t: a = A[g][t], A[g+8][t], A[g][t+4], A[g+8][t+4]; b = B[t][g], B[t+4][g];
// d = D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1])
__device__ __forceinline__ void mma_tf32(float *d, const uint32_t *a, const uint32_t *b)
{
    asm(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Mamba-2 tensor-core row map: accumulator row 16 mt + g + 8 h holds state row
//   srow = 8 g + 4 h + 64 (mt / 4) + mt % 4,
// i.e. 4-row chunk 2 g + h + 16 (mt / 4), row mt % 4 of it.  In the padded chunk layout
// of the slab buffer (chunk c at c (4 VS + 4), row e at e VS) the 4 rows g = 0..3 that a
// half-warp reads together then start 8 banks apart: the float2 fragment reads are free
// of bank conflicts.  Keys and basis rows are indexed with the same map.
__device__ __forceinline__ int srow(int mt, int g, int h) { return 8 * g + 4 * h + 64 * (mt >> 2) + (mt & 3); }
__device__ __forceinline__ int slab_off(int mt, int g, int h, int VS)
{
    return (2 * g + h + 16 * (mt >> 2)) * (4 * VS + 4) + (mt & 3) * VS;
}

__device__ __forceinline__ float2 lds2(const float *p) { return *reinterpret_cast<const float2 *>(p); }
__device__ __forceinline__ void st2(float *p, float a, float b) { *reinterpret_cast<float2 *>(p) = make_float2(a, b); }

// named barrier 1 among the compute warps (the producer warp does not take part)
__device__ __forceinline__ void compute_barrier(int ncw)
{
    asm volatile("bar.sync 1, %0;" ::"r"(ncw * 32) : "memory");
}

// One step of a reduce-scatter between lanes that differ in bit `m`: the lane with
// the bit clear keeps lo (adds the partner's lo), the other keeps hi.
__device__ __forceinline__ float4 rs_step(float4 lo, float4 hi, bool upper, int m)
{
    const float4 keep = upper ? hi : lo, send = upper ? lo : hi;
    return add4(keep, shfl_xor4(send, m));
}

template <int KIND>
__global__ void __launch_bounds__(FLUSH_MAXT, 2)
flush_kernel(const FlushArgs A)
{
    extern __shared__ __align__(128) unsigned char fsm_raw[];
    const int V = A.V, W = A.W, VS = A.VS;
    const int nslab = V / VS;
    const int ncw = VS / 16;  // compute warps
    const FlushCarve cv = flush_carve(KIND, VS, W, A.rcap);
    uint64_t *full = reinterpret_cast<uint64_t *>(fsm_raw + cv.bar);
    uint64_t *empty = full + 1;
    uint64_t *obar = full + 2;
    volatile int *abort = reinterpret_cast<volatile int *>(full + 3);
    float *Sbuf = reinterpret_cast<float *>(fsm_raw + cv.S);
    float *Tb = reinterpret_cast<float *>(fsm_raw + cv.T);
    float *Obuf = reinterpret_cast<float *>(fsm_raw + cv.O);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const long long items = (long long)A.B * A.H * nslab;
    const long long first = items * blockIdx.x / gridDim.x;
    const long long last = items * (blockIdx.x + 1) / gridDim.x;
    if (first >= last) return;
    const int cnt = (int)(last - first);

    if (tid == 0) {
        mbar_init(full, 1);
        mbar_init(empty, ncw);
        mbar_init(obar, 1);
        *abort = 0;
        mbar_fence_init();
    }
    __syncthreads();

    Cursor cur;
    cur.init(A, first, nslab);
    int g_loaded = -1;
    // does this item start a new head group with sketch rows? (tracked alike by all warps)
    auto new_group = [&](const Cursor &c) {
        if (c.r <= 0) return false;
        const int g = c.h / A.Hg;
        if (g == g_loaded) return false;
        g_loaded = g;
        return true;
    };

    if (warp == ncw) {
        // ------------------------------------------------------------ producer
        uint32_t last_full = 0, last_o = 0;
        int issued_o = 0, o_rows = 0;
        auto issue_omega = [&](const Cursor &c) {
            if (lane == 0) {
                const uint32_t bytes = (uint32_t)(o_rows * KDIM * 4);
                mbar_arrive_expect_tx(obar, bytes);
                bulk_copy_g2s(Obuf, A.omega + (long long)(c.h / A.Hg) * A.Rb * KDIM, bytes, obar);
            }
            last_o = (uint32_t)(issued_o & 1);
            ++issued_o;
        };
        // Mamba-2 copies an item's keys only when its key set (b, q/k head) changes: the
        // compute warps read them once, into the fragment cache
        long long pk = (long long)cur.b * A.Hqk + cur.h / A.hpq;
        bool pend_o = new_group(cur);
        if (pend_o) o_rows = __ldg(A.rmax + cur.h / A.Hg);
        issue_item<KIND>(A, cur, nslab, Sbuf, Tb, cv, full, lane, true);
        if (pend_o) issue_omega(cur);
        pend_o = false;
        bool ok = true;
        for (int j = 1; j <= cnt; ++j) {
            // every compute warp holds item j-1's slab and is done with item j-2
            ok = staged_wait(empty, (uint32_t)((j - 1) & 1), A, abort);
            if (!ok) break;
            if (pend_o) issue_omega(cur);  // item j-1's new basis rows
            pend_o = false;
            if (j == cnt) break;
            cur.next(A, nslab);
            pend_o = new_group(cur);
            if (pend_o) o_rows = __ldg(A.rmax + cur.h / A.Hg);  // used one iteration later
            const long long key = (long long)cur.b * A.Hqk + cur.h / A.hpq;
            issue_item<KIND>(A, cur, nslab, Sbuf, Tb + (size_t)(j & 1) * cv.tfloats, cv, full, lane, key != pk);
            pk = key;
            last_full = (uint32_t)(j & 1);
        }
        if (!ok) {
            if (lane == 0) {
                *abort = 1;
                atomicOr(A.status, SK_STATUS_FLUSH_TIMEOUT);
            }
            // copies still in flight land before the CTA's shared memory is released
            mbar_wait_bounded(full, last_full, DEFAULT_WAIT_CYCLES);
            if (issued_o > 0) mbar_wait_bounded(obar, last_o, DEFAULT_WAIT_CYCLES);
        }
        return;
    }

    // ---------------------------------------------------------------- compute warps
    const int ks = lane & 7;
    const int c4 = warp * 4 + (lane >> 3);
    // per-token scalars of the current item in lanes < n
    float a_l = 1.f, b_l = 0.f;
    auto load_scalars = [&](const Cursor &c, float &a, float &bv) {
        a = 1.f;
        bv = 0.f;
        if (lane < c.n) {
            const long long o = c.bh(A) * W + lane;
            if (KIND != SKETCHSSM_KDA) a = __ldg(A.abuf + o);
            if (KIND != SKETCHSSM_MAMBA2) bv = __ldg(A.bbuf + o);
        }
    };
    load_scalars(cur, a_l, b_l);
    uint32_t o_phase = 0;

    if constexpr (KIND == SKETCHSSM_MAMBA2) {
        // ------------------------------------------------ Mamba-2 on the tensor cores
        const int g = lane >> 2, t = lane & 3;
        const int col0 = warp * 16;  // the warp's 16 columns of the slab
        float *AF = reinterpret_cast<float *>(fsm_raw + cv.AF);
        long long af_key = -1;  // (b, q/k head) whose keys the fragment cache holds
        bool ok = true;         // false once a wait gave up: no more work, barriers only
        for (int j = 0; j < cnt; ++j) {
            const float *T = Tb + (size_t)(j & 1) * cv.tfloats;
            const int r = cur.r, n = cur.n;
            const bool need_o = new_group(cur);
            ok = ok && staged_wait(full, (uint32_t)(j & 1), A, abort);
            // the state in the accumulator layout: c[mt][nt][2 h + e] = state row
            // srow(mt, g, h), column col0 + 8 nt + 2 t + e
            float c[8][2][4];
            {
                const float *sb = Sbuf + col0 + 2 * t;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const float2 lo = lds2(sb + slab_off(mt, g, 0, VS) + 8 * nt);
                        const float2 hi = lds2(sb + slab_off(mt, g, 1, VS) + 8 * nt);
                        c[mt][nt][0] = lo.x;
                        c[mt][nt][1] = lo.y;
                        c[mt][nt][2] = hi.x;
                        c[mt][nt][3] = hi.y;
                    }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty);

            Cursor nxt = cur;
            float a_n = 1.f, b_n = 0.f;
            if (j + 1 < cnt) {
                nxt.next(A, nslab);
                load_scalars(nxt, a_n, b_n);
            }

            if (n > 0) {
                // suffix products over the tokens (lanes >= n hold a = 1):
                // x_i = prod_{j >= i} a_j, P = x_0, w_i = x_{i+1} = prod_{j > i} a_j
                float x = a_l;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_down_sync(0xffffffffu, x, o);
                    if (lane + o < 32) x *= y;
                }
                const float P = __shfl_sync(0xffffffffu, x, 0);
                float wl = __shfl_down_sync(0xffffffffu, x, 1);
                if (lane == 31) wl = 1.f;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) c[mt][nt][e] *= P;
                // the keys' A fragments, split hi / lo once per key set (shared by the
                // heads of a q/k head): all compute warps build them between two named
                // barriers; tokens >= n are 0.  Stored [k-step][m-tile][hi | lo][lane][4], so
                // that the 128-bit fragment reads of a warp are 512 consecutive bytes (no
                // bank conflict)
                const long long key = (long long)cur.b * A.Hqk + cur.h / A.hpq;
                if (key != af_key) {
                    af_key = key;
                    compute_barrier(ncw);  // every warp is done with the previous set
                    const int nkt = (n + 7) >> 3;
                    const float *kt = T + cv.tkeys;
                    for (int x = warp * 32 + lane; x < nkt * 8 * 32 * 4; x += ncw * 32) {
                        const int comp = x & 3, ln = (x >> 2) & 31, mt = (x >> 7) & 7, k8 = x >> 10;
                        const int tok = 8 * k8 + (ln & 3) + 4 * (comp >> 1);
                        const float v = (ok && tok < n) ? kt[(size_t)tok * cv.ks + srow(mt, ln >> 2, comp & 1)] : 0.f;
                        uint32_t hi, lo;
                        split_tf32(v, hi, lo);
                        float *f = AF + (size_t)((k8 * 8 + mt) * 64 + ln) * 4;  // lo 128 floats on
                        f[comp] = __uint_as_float(hi);
                        f[128 + comp] = __uint_as_float(lo);
                    }
                    compute_barrier(ncw);
                }
                // S += K^T (w o V), 8 tokens per k-step; tokens >= n contribute 0
                const float *vt = T + cv.tv + col0 + g;
                for (int k0 = 0; k0 < n; k0 += 8) {
                    const int i0 = k0 + t, i1 = k0 + t + 4;
                    const bool ok0 = i0 < n, ok1 = i1 < n;
                    const float w0 = __shfl_sync(0xffffffffu, wl, i0 & 31);
                    const float w1 = __shfl_sync(0xffffffffu, wl, i1 & 31);
                    uint32_t bh[2][2], bl[2][2];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const float v0 = ok0 ? w0 * vt[(size_t)i0 * cv.vs + 8 * nt] : 0.f;
                        const float v1 = ok1 ? w1 * vt[(size_t)i1 * cv.vs + 8 * nt] : 0.f;
                        split_tf32(v0, bh[nt][0], bl[nt][0]);
                        split_tf32(v1, bh[nt][1], bl[nt][1]);
                    }
                    const float *af = AF + (size_t)((k0 >> 3) * 8 * 64 + lane) * 4;
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        const uint4 fh = *reinterpret_cast<const uint4 *>(af + mt * 64 * 4);
                        const uint4 fl = *reinterpret_cast<const uint4 *>(af + mt * 64 * 4 + 128);
                        const uint32_t ah[4] = {fh.x, fh.y, fh.z, fh.w}, al[4] = {fl.x, fl.y, fl.z, fl.w};
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt) {
                            mma_tf32(c[mt][nt], al, bh[nt]);
                            mma_tf32(c[mt][nt], ah, bl[nt]);
                            mma_tf32(c[mt][nt], ah, bh[nt]);
                        }
                    }
                }
                float *Sg = A.S + cur.bh(A) * KDIM * V + (long long)cur.slab * VS + col0 + 2 * t;
                if (ok) {
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt) {
                            st2(Sg + (long long)srow(mt, g, 0) * V + 8 * nt, c[mt][nt][0], c[mt][nt][1]);
                            st2(Sg + (long long)srow(mt, g, 1) * V + 8 * nt, c[mt][nt][2], c[mt][nt][3]);
                        }
                }
            }

            // the sketch rows of the warp's columns, 8 at a time: partial sums over the
            // thread's 16 state rows, then a reduce-scatter over g (lane bits 2..4)
            // leaves sketch row m0 + g in lane 4 g + t
            if (need_o) {
                ok = ok && staged_wait(obar, o_phase, A, abort);
                o_phase ^= 1u;
            }
            if (cur.proj && ok) {
                float *Yh = A.Y + ((long long)cur.b * A.rtot + cur.off) * V + (long long)cur.slab * VS + col0 + 2 * t;
                const float *om = Obuf;
                for (int m0 = 0; m0 < r; m0 += 8) {
                    float4 p[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        float4 x0 = zero4(), x1 = zero4();
                        if (m0 + u < r) {
                            // the thread's 16 rows 8 g + 4 h + 64 (mt / 4) + mt % 4 are two
                            // runs of 8 floats: four float4 reads
                            const float *o = om + (m0 + u) * KDIM + 8 * g;
                            const float4 oq[4] = {lds4(o), lds4(o + 4), lds4(o + 64), lds4(o + 68)};
                            const float ov[4][4] = {{oq[0].x, oq[0].y, oq[0].z, oq[0].w},
                                                    {oq[1].x, oq[1].y, oq[1].z, oq[1].w},
                                                    {oq[2].x, oq[2].y, oq[2].z, oq[2].w},
                                                    {oq[3].x, oq[3].y, oq[3].z, oq[3].w}};
#pragma unroll
                            for (int mt = 0; mt < 8; ++mt) {
                                const float o0 = ov[2 * (mt >> 2)][mt & 3], o1 = ov[2 * (mt >> 2) + 1][mt & 3];
                                float4 &xx = (mt & 1) ? x1 : x0;
                                xx.x = fmaf(o0, c[mt][0][0], xx.x);
                                xx.y = fmaf(o0, c[mt][0][1], xx.y);
                                xx.z = fmaf(o0, c[mt][1][0], xx.z);
                                xx.w = fmaf(o0, c[mt][1][1], xx.w);
                                xx.x = fmaf(o1, c[mt][0][2], xx.x);
                                xx.y = fmaf(o1, c[mt][0][3], xx.y);
                                xx.z = fmaf(o1, c[mt][1][2], xx.z);
                                xx.w = fmaf(o1, c[mt][1][3], xx.w);
                            }
                        }
                        p[u] = add4(x0, x1);
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) p[u] = rs_step(p[u], p[u + 4], (lane & 16) != 0, 16);
#pragma unroll
                    for (int u = 0; u < 2; ++u) p[u] = rs_step(p[u], p[u + 2], (lane & 8) != 0, 8);
                    p[0] = rs_step(p[0], p[1], (lane & 4) != 0, 4);
                    if (m0 + g < r) {
                        float *y = Yh + (long long)(m0 + g) * V;
                        st2(y, p[0].x, p[0].y);
                        st2(y + 8, p[0].z, p[0].w);
                    }
                }
            }
            cur = nxt;
            a_l = a_n;
            b_l = b_n;
        }
        if (!ok && lane == 0) {
            *abort = 1;
            atomicOr(A.status, SK_STATUS_FLUSH_TIMEOUT);
        }
    } else {
        for (int j = 0; j < cnt; ++j) {
            const float *T = Tb + (size_t)(j & 1) * cv.tfloats;
            const int r = cur.r, n = cur.n;
            const bool need_o = new_group(cur);

            if (!staged_wait(full, (uint32_t)(j & 1), A, abort)) {
                if (lane == 0) {
                    *abort = 1;
                    atomicOr(A.status, SK_STATUS_FLUSH_TIMEOUT);
                }
                return;
            }
            float4 s[16];
            {
                const float *sb = Sbuf + (size_t)ks * (4 * VS + 4) + c4 * 4;
#pragma unroll
                for (int q = 0; q < QROWS; ++q)
#pragma unroll
                    for (int e = 0; e < 4; ++e) s[4 * q + e] = lds4(sb + (size_t)q * 8 * (4 * VS + 4) + e * VS);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty);

            // the next item's scalars, one item ahead
            Cursor nxt = cur;
            float a_n = 1.f, b_n = 0.f;
            if (j + 1 < cnt) {
                nxt.next(A, nslab);
                load_scalars(nxt, a_n, b_n);
            }

            // the update
            const float *kt = T + cv.tkeys + 4 * ks;
            const float *vt = T + cv.tv + c4 * 4;
            const float *at = T + cv.ta + 4 * ks;
            for (int i = 0; i < n; ++i) {
                const float *ki = kt + i * KDIM;
                float4 kq[QROWS];
#pragma unroll
                for (int q = 0; q < QROWS; ++q) kq[q] = lds4(ki + q * 32);
                float4 d0 = zero4(), d1 = zero4();
                quad_dot(d0, kq[0], s + 0);
                quad_dot(d1, kq[1], s + 4);
                quad_dot(d0, kq[2], s + 8);
                quad_dot(d1, kq[3], s + 12);
                const float4 d = sum8_xor(add4(d0, d1));  // d = S^T k_i for this column chunk
                const float4 vv = lds4(vt + i * VS);
                const float bi = __shfl_sync(0xffffffffu, b_l, i);
                if (KIND == SKETCHSSM_GDN) {
                    // a (S - beta k d) + beta k v = a S + k * beta (v - a d)
                    const float ai = __shfl_sync(0xffffffffu, a_l, i);
                    const float4 u = make_float4(bi * fmaf(-ai, d.x, vv.x), bi * fmaf(-ai, d.y, vv.y),
                                                 bi * fmaf(-ai, d.z, vv.z), bi * fmaf(-ai, d.w, vv.w));
#pragma unroll
                    for (int q = 0; q < QROWS; ++q) {
                        const float kk[4] = {kq[q].x, kq[q].y, kq[q].z, kq[q].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float4 &t = s[4 * q + e];
                            t.x = fmaf(ai, t.x, kk[e] * u.x);
                            t.y = fmaf(ai, t.y, kk[e] * u.y);
                            t.z = fmaf(ai, t.z, kk[e] * u.z);
                            t.w = fmaf(ai, t.w, kk[e] * u.w);
                        }
                    }
                } else {
                    // a_k (S - beta k_k d) + beta k_k v = a_k S + beta k_k (v - a_k d)
                    const float *ai = at + i * KDIM;
#pragma unroll
                    for (int q = 0; q < QROWS; ++q) {
                        const float4 a4 = lds4(ai + q * 32);
                        const float kk[4] = {kq[q].x, kq[q].y, kq[q].z, kq[q].w};
                        const float aq[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float4 &t = s[4 * q + e];
                            const float ak = aq[e], kb = bi * kk[e];
                            t.x = fmaf(ak, t.x, kb * fmaf(-ak, d.x, vv.x));
                            t.y = fmaf(ak, t.y, kb * fmaf(-ak, d.y, vv.y));
                            t.z = fmaf(ak, t.z, kb * fmaf(-ak, d.z, vv.z));
                            t.w = fmaf(ak, t.w, kb * fmaf(-ak, d.w, vv.w));
                        }
                    }
                }
            }
            const long long bh = cur.bh(A);
            if (n > 0) {
                float *Sg = A.S + (bh * KDIM + 4 * ks) * V + (long long)cur.slab * VS + c4 * 4;
#pragma unroll
                for (int q = 0; q < QROWS; ++q)
#pragma unroll
                    for (int e = 0; e < 4; ++e) st4(Sg + (long long)(32 * q + e) * V, s[4 * q + e]);
            }

            // the sketch rows of this slab: 8 rows at a time, reduced over the 8 row slices
            // by a reduce-scatter that leaves row m0 + ks in lane ks
            if (need_o) {
                if (!staged_wait(obar, o_phase, A, abort)) {
                    if (lane == 0) {
                        *abort = 1;
                        atomicOr(A.status, SK_STATUS_FLUSH_TIMEOUT);
                    }
                    return;
                }
                o_phase ^= 1u;
            }
            if (cur.proj) {
                float *Yh = A.Y + ((long long)cur.b * A.rtot + cur.off) * V + (long long)cur.slab * VS +
                            c4 * 4;
                const float *om = Obuf + 4 * ks;
                const bool u2 = ks & 4, u1 = ks & 2, u0 = ks & 1;
                for (int m0 = 0; m0 < r; m0 += 8) {
                    float4 p[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        float4 x0 = zero4(), x1 = zero4();
                        if (m0 + u < r) {
                            const float *o = om + (m0 + u) * KDIM;
                            quad_dot(x0, lds4(o), s + 0);
                            quad_dot(x1, lds4(o + 32), s + 4);
                            quad_dot(x0, lds4(o + 64), s + 8);
                            quad_dot(x1, lds4(o + 96), s + 12);
                        }
                        p[u] = add4(x0, x1);
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) p[u] = rs_step(p[u], p[u + 4], u2, 4);
#pragma unroll
                    for (int u = 0; u < 2; ++u) p[u] = rs_step(p[u], p[u + 2], u1, 2);
                    p[0] = rs_step(p[0], p[1], u0, 1);
                    if (m0 + ks < r) st4(Yh + (long long)(m0 + ks) * V, p[0]);
                }
            }
            cur = nxt;
            a_l = a_n;
            b_l = b_n;
        }
    }
}

template <int KIND>
cudaError_t launch_kind(const FlushArgs &a, cudaStream_t stream)
{
    const FlushCarve cv = flush_carve(KIND, a.VS, a.W, a.rcap);
    const int threads = 32 * (a.VS / 16 + 1);
    auto kern = flush_kernel<KIND>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cv.total);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, cv.total)) != cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const long long items = (long long)a.B * a.H * (a.V / a.VS);
    long long grid = (long long)per_sm * sms;
    if (grid > items) grid = items;
    kern<<<(unsigned)grid, threads, cv.total, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

int flush_slab(int V)
{
    // up to 80 columns in one slab; wider states in slabs of at most 64 columns, so
    // that the slab buffer, two token buffers and the basis rows fit shared memory
    if (V <= 80) return V;
    for (int vs = 64; vs >= 16; vs -= 16)
        if (V % vs == 0) return vs;
    return 16;
}

size_t flush_smem_bytes(int kind, int V, int W, int rcap)
{
    return flush_carve(kind, flush_slab(V), W, rcap).total;
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
