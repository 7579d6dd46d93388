// Mamba-2 prefill on the 5th-generation tensor cores (tcgen05, accumulator in tensor
// memory).
//
// Paper abstract (SketchSSM, newx.sg / mlsanity pages): every state update reaches the
// full state.  A prompt of T tokens applied to a Mamba-2 state token after token,
// S <- a_t S + k_t v_t^T, unrolls to one contraction
//
//     S_T = G S_0 + sum_t w_t k_t v_t^T,   w_t = prod_{t<j<T} a_j,   G = prod_{j<T} a_j,
//
// taken transposed, D^T[n][m] = sum_t (w_t v_t[n]) k_t[m], so that tensor-memory lane n
// holds value column n of the new state.
//
// One CTA of 128 threads per (batch row, q/k head) walks that q/k head's heads, two CTAs
// per SM.  The prompt's keys (shared by the heads) are staged once as the B operand
// (N = 128 state rows); each head's weighted values w_t v_t[n] are the A operand (M = 128
// rows: rows n >= V read whatever follows them and land in lanes nobody reads); one
// thread of the last warp issues the MMAs (K = 8 tokens a step) into one of two
// tensor-memory accumulators.  So the MMAs of head j run while the epilogue of head
// j - 1 proceeds: thread n (lane n) adds G S_0[m][n] to D^T[n][m], 16 state rows m at a
// time, and its warp writes each state row as 128 contiguous bytes.  Meanwhile the
// loads for head j + 1 (its values) and head j (its S_0 column) are in flight into
// registers.
//
// Precision: every operand x is split into hi = x with its 13 low mantissa bits cleared
// (exact in tf32) and lo = x - hi (exact in fp32), and D accumulates hi*hi + hi*lo +
// lo*hi in fp32: the products lose only lo*lo and the tf32 truncation of lo, about
// 2^-21 relative, well inside the 1e-4 parity bound.
//
// Operand tiles are K-major without swizzling: element (r, t) of an R-row tile sits in
// the 8-row x 16-byte core matrix (r / 8, t / 4) at byte ((t / 4) R / 8 + r / 8) 128 +
// (r % 8) 16 + (t % 4) 4, so that a thread writing 4 consecutive tokens of row r writes
// 16 contiguous bytes and a warp's 32 rows 512 contiguous bytes.
#include "device_util.cuh"
#include "internal.cuh"
#include "ptx_util.cuh"

namespace sk {
namespace {

constexpr int PU_THREADS = 128;  // one thread per tensor-memory lane (value column)
constexpr int PU_TMAX = 64;      // prompt tokens staged at once (longer prompts take the other kernel)

__host__ __device__ constexpr int pu_round8(int x) { return (x + 7) & ~7; }

struct PuCarve {
    size_t kh, kl, vh, vl, w, g, bar, taddr, total;
};

__host__ __device__ inline size_t pu_take(size_t &o, size_t bytes)
{
    const size_t r = o;
    o = (o + bytes + 127) & ~size_t(127);
    return r;
}

__host__ __device__ inline PuCarve pu_carve(int V, int tp)
{
    PuCarve c;
    size_t o = 0;
    c.kh = pu_take(o, sizeof(float) * KDIM * (size_t)tp);
    c.kl = pu_take(o, sizeof(float) * KDIM * (size_t)tp);
    c.vh = pu_take(o, sizeof(float) * (size_t)V * tp);
    c.vl = pu_take(o, sizeof(float) * (size_t)V * tp + 16 * (size_t)(KDIM - V));  // rows V..127 of the last quad read past it
    c.w = pu_take(o, sizeof(float) * PU_TMAX);
    c.g = pu_take(o, sizeof(float) * 2);
    c.bar = pu_take(o, sizeof(uint64_t) * 2);
    c.taddr = pu_take(o, sizeof(uint32_t));
    c.total = o;
    return c;
}


__device__ __forceinline__ float tf32_hi(float x)
{
    return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
}

// hi and lo parts of 4 values to the two tiles (16 bytes each)
__device__ __forceinline__ void put_split(float *hi, float *lo, size_t off, float4 x)
{
    const float4 h = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
    st4(hi + off, h);
    st4(lo + off, make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w));
}

// All threads wait for phase `parity` of `bar` (the CTA's own MMAs).  A wait past the
// plan's limit is recorded (sketchssm_plan_check reports it) and continued up to
// DEFAULT_WAIT_CYCLES; false only if that runs out too.
__device__ __forceinline__ bool pu_wait(const PrefillArgs &A, uint64_t *bar, uint32_t parity)
{
    bool ok = mbar_wait_bounded(bar, parity, A.wait_limit);
    if (!__syncthreads_or(!ok)) return true;
    if (threadIdx.x == 0) atomicOr(A.status, SK_STATUS_PREFILL_TIMEOUT);
    ok = mbar_wait_bounded(bar, parity, DEFAULT_WAIT_CYCLES);
    return !__syncthreads_or(!ok);
}

template <int V>
__global__ void __launch_bounds__(PU_THREADS, 2) prefill_tcgen05_kernel(const PrefillArgs A)
{
    constexpr int TASKS = (V * (PU_TMAX / 4) + PU_THREADS - 1) / PU_THREADS;  // B-tile quads a thread builds
    extern __shared__ __align__(1024) unsigned char pus[];
    const int T = A.T, tp = pu_round8(T), nq = tp / 4;
    const PuCarve cv = pu_carve(V, tp);
    float *kh = reinterpret_cast<float *>(pus + cv.kh), *kl = reinterpret_cast<float *>(pus + cv.kl);
    float *vh = reinterpret_cast<float *>(pus + cv.vh), *vl = reinterpret_cast<float *>(pus + cv.vl);
    float *w_s = reinterpret_cast<float *>(pus + cv.w);
    float *g_s = reinterpret_cast<float *>(pus + cv.g);
    uint64_t *bar = reinterpret_cast<uint64_t *>(pus + cv.bar);
    uint32_t *taddr = reinterpret_cast<uint32_t *>(pus + cv.taddr);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int qk = blockIdx.x, b = blockIdx.y, H = A.H, nh = A.hpq, h0 = qk * nh;
    const long long tok0 = (long long)b * T;  // token 0 of row b
    constexpr uint32_t COLS = 2 * KDIM;  // two accumulators of 128 columns (one per state row)

    if (warp == 0) {
        tmem_alloc(taddr, COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 1, 1);
        mbar_fence_init();
    }

    // loads for head j: its decays (thread t) and raw values (B-tile quads of this thread)
    float a_r = 1.f, a_r2 = 1.f;  // warp 0: the decays of tokens lane and 32 + lane (1 past T)
    float4 vr[TASKS];
    auto load_head = [&](int j) {
        const int h = h0 + j;
        if (warp == 0) {
            a_r = tid < T ? __ldg(A.a + (tok0 + tid) * H + h) : 1.f;
            a_r2 = tid + 32 < T ? __ldg(A.a + (tok0 + tid + 32) * H + h) : 1.f;
        }
#pragma unroll
        for (int u = 0; u < TASKS; ++u) {
            const int x = tid + u * PU_THREADS, n = x % V, q = x / V;
            float4 r = zero4();
            if (q < nq) {
                const float *vp = A.v + ((tok0 + 4 * q) * H + h) * V + n;
                const long long st = (long long)H * V;
                if (4 * q + 0 < T) r.x = __ldg(vp);
                if (4 * q + 1 < T) r.y = __ldg(vp + st);
                if (4 * q + 2 < T) r.z = __ldg(vp + 2 * st);
                if (4 * q + 3 < T) r.w = __ldg(vp + 3 * st);
            }
            vr[u] = r;
        }
    };
    load_head(0);

    // the prompt's keys, once: thread m holds state row m, 4 tokens at a time
    for (int q = 0; q < nq; ++q) {
        float4 x = zero4();
        const float *kp = A.k + ((tok0 + 4 * q) * A.Hqk + qk) * KDIM + tid;
        const long long st = (long long)A.Hqk * KDIM;
        if (4 * q + 0 < T) x.x = __ldg(kp);
        if (4 * q + 1 < T) x.y = __ldg(kp + st);
        if (4 * q + 2 < T) x.z = __ldg(kp + 2 * st);
        if (4 * q + 3 < T) x.w = __ldg(kp + 3 * st);
        put_split(kh, kl, ((size_t)q * KDIM + tid) * 4, x);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *taddr;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    // D^T[n][m] = sum_t (w_t v_t[n]) k_t[m]: A = the weighted values (M = 128 rows, rows
    // n >= V read whatever follows them and land in accumulator lanes nobody reads),
    // B = the keys (N = 128 state rows), so that lane n of tensor memory holds column n
    // of the new state and a warp's stores of one state row are 128 contiguous bytes
    const uint32_t idesc = umma_idesc_tf32(128, KDIM);
    const int n_own = warp * 32 + (tid & 31);  // the state column this thread writes back
    const bool epi_warp = warp * 32 < V;      // warps holding at least one column
    const bool own = n_own < V;

    float s0[KDIM];  // S_0 column n_own of the head whose epilogue comes next
    bool ok = true;
    int jw = 0;     // the head whose products a wait gave up on
    for (int j = 0; j <= nh && ok; ++j) {
        const int buf = j & 1;
        if (j < nh) {
            // decay weights of head j, w_t = prod_{t<i<T} a_i and G = prod_i a_i: warp 0
            // holds tokens 2 l, 2 l + 1 in lane l and takes suffix products over the lanes
            if (warp == 0) {
                const int l = tid;
                const float a0 = __shfl_sync(0xffffffffu, a_r, (2 * l) & 31), a1 = __shfl_sync(0xffffffffu, a_r, (2 * l + 1) & 31);
                const float b0 = __shfl_sync(0xffffffffu, a_r2, (2 * l) & 31), b1 = __shfl_sync(0xffffffffu, a_r2, (2 * l + 1) & 31);
                const float x0 = l < 16 ? a0 : b0, x1 = l < 16 ? a1 : b1;  // a_{2l}, a_{2l+1} (1 past T)
                float p = x0 * x1;  // inclusive suffix product over pairs l .. 31
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const float o = __shfl_down_sync(0xffffffffu, p, d);
                    if (l + d < 32) p *= o;
                }
                float after = __shfl_down_sync(0xffffffffu, p, 1);  // pairs l + 1 .. 31
                if (l == 31) after = 1.f;
                const float w1 = after, w0 = x1 * after;  // w_{2l+1}, w_{2l}
                if (2 * l < tp) w_s[2 * l] = 2 * l < T ? w0 : 0.f;
                if (2 * l + 1 < tp) w_s[2 * l + 1] = 2 * l + 1 < T ? w1 : 0.f;
                if (l == 0) g_s[buf] = p;
            }
        }
        // head j - 1's products have landed: its accumulator is ready and the values tile free
        if (j >= 1 && !(ok = pu_wait(A, bar + ((j - 1) & 1), ((j - 1) >> 1) & 1))) {
            jw = j - 1;
            break;
        }
        tc_fence_after();
        __syncthreads();  // w_s, g_s
        if (j < nh) {
            // head j's values tile: quad (n, q) = w_t v_t[n] for the 4 tokens of quad q
#pragma unroll
            for (int u = 0; u < TASKS; ++u) {
                const int x = tid + u * PU_THREADS, n = x % V, q = x / V;
                if (q < nq) {
                    const float4 wq = lds4(w_s + 4 * q);
                    const float4 r = vr[u];
                    put_split(vh, vl, ((size_t)q * V + n) * 4,
                              make_float4(wq.x * r.x, wq.y * r.y, wq.z * r.z, wq.w * r.w));
                }
            }
            if (j + 1 < nh) load_head(j + 1);
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (tid == PU_THREADS - 32) {
                // one thread of the last warp issues (it blocks while the tensor core's
                // queue is full; the last warp holds no state column when V <= 96, so
                // the others start their epilogue meanwhile)
                // tokens 8 s .. 8 s + 7: core columns 2 s, 2 s + 1 of each tile
                const uint32_t d = tmem + (uint32_t)(buf * KDIM);
                int c = 0;
                for (int s = 0; s < tp / 8; ++s) {
                    const uint32_t ka = (uint32_t)s * 2 * KDIM * 16, vb = (uint32_t)s * 2 * V * 16;
                    const uint64_t ah = umma_sdesc(smem_addr(vh) + vb, V * 16, 128);
                    const uint64_t al = umma_sdesc(smem_addr(vl) + vb, V * 16, 128);
                    const uint64_t bh = umma_sdesc(smem_addr(kh) + ka, KDIM * 16, 128);
                    const uint64_t bl = umma_sdesc(smem_addr(kl) + ka, KDIM * 16, 128);
                    umma_tf32(d, ah, bh, idesc, c++ > 0);
                    umma_tf32(d, ah, bl, idesc, 1u);
                    umma_tf32(d, al, bh, idesc, 1u);
                }
                umma_commit(bar + buf);
            }
        }
        if (j >= 1 && epi_warp) {
            // epilogue of head j - 1: S_T[m][n] = D^T[n][m] + G S_0[m][n], 16 rows m at a time
            const int h = h0 + j - 1;
            const float g = g_s[(j - 1) & 1];
            float *Sc = A.S + ((long long)b * H + h) * KDIM * V + n_own;
            const uint32_t d = tmem + lane_base + (uint32_t)(((j - 1) & 1) * KDIM);
#pragma unroll
            for (int m0 = 0; m0 < KDIM; m0 += 16) {
                float x[16];
                tmem_ld16(d + m0, x);
                if (own) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) Sc[(long long)(m0 + e) * V] = fmaf(g, s0[m0 + e], x[e]);
                }
            }
        }
        if (j < nh && own) {
            // S_0 of head j, for its epilogue in the next round
            const float *S0 = A.S + ((long long)b * H + h0 + j) * KDIM * V + n_own;
#pragma unroll
            for (int m = 0; m < KDIM; ++m) s0[m] = __ldg(S0 + (long long)m * V);
        }
        tc_fence_before();
    }
    if (!ok && tid == 0) {
        // a wait gave up: let that head's MMAs (the only ones in flight) finish, bounded,
        // before the tensor memory is released
        mbar_wait_bounded(bar + (jw & 1), (jw >> 1) & 1, DEFAULT_WAIT_CYCLES);
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, COLS);
}

template <int V>
cudaError_t launch_v(const PrefillArgs &a, cudaStream_t stream)
{
    const PuCarve cv = pu_carve(V, pu_round8(a.T));
    // at least 80 KB, so that at most two CTAs share an SM and their tensor-memory
    // allocations (256 columns each) always fit the SM's 512 columns
    const size_t smem = cv.total > 80 * 1024 ? cv.total : 80 * 1024;
    cudaError_t e = cudaFuncSetAttribute(prefill_tcgen05_kernel<V>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    prefill_tcgen05_kernel<V><<<dim3(a.Hqk, a.B), PU_THREADS, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool prefill_tcgen05_fits(const PrefillArgs &a)
{
    return a.kind == SKETCHSSM_MAMBA2 && a.T >= 1 && a.T <= PU_TMAX && a.V % 16 == 0 && a.V >= 16 && a.V <= 128 &&
           a.Hqk <= 65535 && a.B <= 65535;
}

cudaError_t launch_prefill_tcgen05(const PrefillArgs &a, cudaStream_t stream)
{
    switch (a.V) {
    case 16: return launch_v<16>(a, stream);
    case 32: return launch_v<32>(a, stream);
    case 48: return launch_v<48>(a, stream);
    case 64: return launch_v<64>(a, stream);
    case 80: return launch_v<80>(a, stream);
    case 96: return launch_v<96>(a, stream);
    case 112: return launch_v<112>(a, stream);
    default: return launch_v<128>(a, stream);
    }
}

}  // namespace sk
