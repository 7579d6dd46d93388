// Host side of the C ABI declared in include/sketchssm.h: argument checks, the
// plan (device rank / offset / work tables built by the layout kernel), and the
// launches of the flush, sketch-decode and dense-read decode kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <string>

#include "internal.cuh"

namespace {

thread_local std::string g_last_error;

sketchssm_status fail(sketchssm_status s, const std::string &msg)
{
    g_last_error = msg;
    return s;
}

sketchssm_status cuda_fail(cudaError_t e, const char *what)
{
    g_last_error = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
    return SKETCHSSM_ERR_CUDA;
}

// cuMemGetAddressRange through the runtime's driver entry point, so the library does
// not link libcuda itself.
typedef CUresult (*AddrRangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);

AddrRangeFn addr_range_fn()
{
    static AddrRangeFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return (AddrRangeFn) nullptr;
        }
        return (AddrRangeFn)p;
    }();
    return fn;
}

// A tensor argument must be 16-byte aligned device memory (of the current device,
// or managed / mapped host memory) whose allocation holds `bytes` from `p` on.
sketchssm_status check_tensor(const void *p, size_t bytes, const char *name, bool may_be_null)
{
    if (p == nullptr) {
        if (may_be_null || bytes == 0) return SKETCHSSM_OK;
        return fail(SKETCHSSM_ERR_INVALID_ARG, std::string(name) + " is NULL");
    }
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0)
        return fail(SKETCHSSM_ERR_ALIGNMENT, std::string(name) + " is not 16-byte aligned");
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(SKETCHSSM_ERR_INVALID_ARG, std::string(name) + " is not a CUDA pointer");
    }
    if (at.type == cudaMemoryTypeUnregistered ||
        (at.type == cudaMemoryTypeHost && at.devicePointer == nullptr))
        return fail(SKETCHSSM_ERR_INVALID_ARG, std::string(name) + " is not device-accessible memory");
    if (at.type == cudaMemoryTypeDevice) {
        int dev = -1;
        cudaGetDevice(&dev);
        if (at.device != dev)
            return fail(SKETCHSSM_ERR_INVALID_ARG, std::string(name) + " lives on another device");
        if (AddrRangeFn fn = addr_range_fn()) {
            CUdeviceptr base = 0;
            size_t size = 0;
            if (fn(&base, &size, (CUdeviceptr)p) == CUDA_SUCCESS) {
                const size_t avail = (size_t)(base + size - (CUdeviceptr)p);
                if (bytes > avail)
                    return fail(SKETCHSSM_ERR_INVALID_ARG,
                                std::string(name) + " allocation is smaller than the tensor (" +
                                    std::to_string(avail) + " < " + std::to_string(bytes) + " bytes)");
            }
        }
    }
    return SKETCHSSM_OK;
}

#define CHECK_T(ptr, bytes, name, nullable)                                    \
    do {                                                                       \
        sketchssm_status s_ = check_tensor((ptr), (bytes), (name), (nullable)); \
        if (s_ != SKETCHSSM_OK) return s_;                                     \
    } while (0)

sketchssm_status check_desc(const sketchssm_desc *d)
{
    if (!d) return fail(SKETCHSSM_ERR_INVALID_ARG, "desc is NULL");
    if (d->kind < SKETCHSSM_MAMBA2 || d->kind > SKETCHSSM_KDA)
        return fail(SKETCHSSM_ERR_INVALID_ARG, "unknown kind");
    if (d->batch < 1 || d->heads < 1 || d->qk_heads < 1 || d->groups < 1 || d->window < 1 ||
        d->key_dim < 1 || d->value_dim < 1 || d->basis_rows < 1 || d->rank_cap < 1)
        return fail(SKETCHSSM_ERR_INVALID_ARG, "every size in desc must be >= 1");
    if (d->heads % d->groups != 0) return fail(SKETCHSSM_ERR_INVALID_ARG, "heads % groups != 0");
    if (d->heads % d->qk_heads != 0) return fail(SKETCHSSM_ERR_INVALID_ARG, "heads % qk_heads != 0");
    if (d->basis_rows > d->key_dim) return fail(SKETCHSSM_ERR_INVALID_ARG, "basis_rows > key_dim");
    if (d->rank_cap > d->basis_rows) return fail(SKETCHSSM_ERR_INVALID_ARG, "rank_cap > basis_rows");
    if (d->key_dim != sk::KDIM) return fail(SKETCHSSM_ERR_UNSUPPORTED, "key_dim must be 128");
    if (d->value_dim % 16 != 0 || d->value_dim > sk::MAX_V)
        return fail(SKETCHSSM_ERR_UNSUPPORTED, "value_dim must be a multiple of 16 in [16, 256]");
    if (d->window > sk::MAX_W) return fail(SKETCHSSM_ERR_UNSUPPORTED, "window must be <= 32");
    if (d->heads / d->groups > sk::MAX_HG) return fail(SKETCHSSM_ERR_UNSUPPORTED, "heads/groups must be <= 32");
    if (d->qk_heads % d->groups != 0)
        return fail(SKETCHSSM_ERR_UNSUPPORTED, "qk_heads must be a multiple of groups");
    if (d->heads > (1 << 24)) return fail(SKETCHSSM_ERR_UNSUPPORTED, "too many heads");
    return SKETCHSSM_OK;
}

sketchssm_status check_plan(const sketchssm_plan *p)
{
    if (!p) return fail(SKETCHSSM_ERR_INVALID_ARG, "plan is NULL");
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != p->device) return fail(SKETCHSSM_ERR_INVALID_ARG, "plan was created on another device");
    return SKETCHSSM_OK;
}

size_t fbytes(long long a, long long b = 1, long long c = 1, long long d = 1)
{
    return (size_t)(a * b * c * d) * sizeof(float);
}

sk::DecodeArgs decode_args(const sketchssm_plan *p, int pos, const float *q, const float *k,
                           const float *v, const float *a, const float *beta, float *kbuf,
                           float *vbuf, float *abuf, float *bbuf, const float *Y,
                           const float *omega, const float *S, float *y, int dense_all)
{
    const sketchssm_desc &d = p->d;
    sk::DecodeArgs A;
    A.kind = d.kind;
    A.B = d.batch;
    A.H = d.heads;
    A.Hqk = d.qk_heads;
    A.V = d.value_dim;
    A.W = d.window;
    A.G = d.groups;
    A.Rb = d.basis_rows;
    A.cap = d.rank_cap;
    A.pos = pos;
    A.Hg = p->Hg;
    A.hpq = p->hpq;
    A.rtot = p->rtot;
    A.rank = p->d_rank;
    A.off = p->d_off;
    A.coff = p->d_coff;
    A.coef_dense_block = sk::coef_block(sk::KDIM, d.window);
    A.coef_row = dense_all ? d.heads * A.coef_dense_block : p->coef_row;
    A.scratch = p->d_scratch;
    A.work = p->d_work + (size_t)pos * (d.heads + d.groups);
    A.rec = p->d_rec + (size_t)pos * (d.heads + d.groups) * 8;
    A.qk_rneed = p->d_qk_rneed;
    A.n_items = dense_all ? d.heads : p->h_items[pos];
    A.dense_all = dense_all;
    A.threads = p->geo.threads;
    A.stage_rows = p->geo.stage_rows;
    A.cm_rows = sk::coef_rows(d.rank_cap, d.window, d.batch, d.qk_heads, p->sms);
    A.dots_row = sk::dots_row(d.window, d.rank_cap);
    A.maxnh = p->geo.maxnh;
    A.coef_cap = p->geo.coef_cap;
    A.wait_limit = p->wait_limit;
    A.status = p->d_status;
    A.row_pos = nullptr;
    A.counts = p->d_counts;
    A.q = q;
    A.k = k;
    A.v = v;
    A.a = a;
    A.beta = beta;
    A.kbuf = kbuf;
    A.vbuf = vbuf;
    A.abuf = abuf;
    A.bbuf = bbuf;
    A.Y = Y;
    A.omega = omega;
    A.S = S;
    A.y = y;
    return A;
}

sketchssm_status check_decode_common(const sketchssm_plan *p, int pos, const float *q, const float *k,
                                     const float *v, const float *a, const float *beta,
                                     const float *kbuf, const float *vbuf, const float *abuf,
                                     const float *bbuf, const float *y)
{
    const sketchssm_desc &d = p->d;
    if (pos < 0 || pos >= d.window) return fail(SKETCHSSM_ERR_INVALID_ARG, "pos outside [0, window)");
    const long long B = d.batch, H = d.heads, Q = d.qk_heads, K = d.key_dim, V = d.value_dim,
                    W = d.window;
    const long long da = d.kind == SKETCHSSM_KDA ? K : 1;
    const bool mamba = d.kind == SKETCHSSM_MAMBA2;
    CHECK_T(q, fbytes(B, Q, K), "q", false);
    CHECK_T(k, fbytes(B, Q, K), "k", false);
    CHECK_T(v, fbytes(B, H, V), "v", false);
    CHECK_T(a, fbytes(B, H, da), "a", false);
    CHECK_T(beta, mamba ? 0 : fbytes(B, H), "beta", mamba);
    CHECK_T(kbuf, fbytes(B, Q, W, K), "kbuf", false);
    CHECK_T(vbuf, fbytes(B, H, W, V), "vbuf", false);
    CHECK_T(abuf, fbytes(B, H, W, da), "abuf", false);
    CHECK_T(bbuf, mamba ? 0 : fbytes(B, H, W), "bbuf", mamba);
    CHECK_T(y, fbytes(B, H, V), "y", false);
    return SKETCHSSM_OK;
}

}  // namespace

extern "C" {

const char *sketchssm_status_string(sketchssm_status s)
{
    switch (s) {
    case SKETCHSSM_OK: return "ok";
    case SKETCHSSM_ERR_INVALID_ARG: return "invalid argument";
    case SKETCHSSM_ERR_ALIGNMENT: return "misaligned tensor";
    case SKETCHSSM_ERR_UNSUPPORTED: return "unsupported shape";
    case SKETCHSSM_ERR_CUDA: return "CUDA error";
    case SKETCHSSM_ERR_TIMEOUT: return "timeout";
    }
    return "unknown status";
}

const char *sketchssm_last_error(void) { return g_last_error.c_str(); }

sketchssm_status sketchssm_plan_create(const sketchssm_desc *desc, const int32_t *rank_host,
                                       const int32_t *group_host, sketchssm_stream stream,
                                       sketchssm_plan **out)
{
    g_last_error.clear();
    if (!out) return fail(SKETCHSSM_ERR_INVALID_ARG, "out is NULL");
    sketchssm_status s = check_desc(desc);
    if (s != SKETCHSSM_OK) return s;
    if (!rank_host) return fail(SKETCHSSM_ERR_INVALID_ARG, "rank table is NULL");
    const sketchssm_desc d = *desc;
    const int H = d.heads, G = d.groups;
    if (group_host) {
        // the kernels are built for contiguous groups of H/G heads
        for (int h = 0; h < H; ++h) {
            const int g = group_host[h];
            if (g < 0 || g >= G)
                return fail(SKETCHSSM_ERR_INVALID_ARG, "group[" + std::to_string(h) + "] = " + std::to_string(g) +
                                                           " is outside [0, groups)");
        }
        for (int h = 0; h < H; ++h)
            if (group_host[h] != h / (H / G))
                return fail(SKETCHSSM_ERR_UNSUPPORTED,
                            "group[" + std::to_string(h) + "] = " + std::to_string(group_host[h]) +
                                ": only contiguous groups (head h in group h / (heads / groups)) are supported; "
                                "number the heads group by group");
    }
    long long rtot = 0;
    for (int h = 0; h < H; ++h) {
        const int r = rank_host[h];
        if (r == SKETCHSSM_DENSE) continue;
        if (r < 1 || r > d.rank_cap)
            return fail(SKETCHSSM_ERR_INVALID_ARG,
                        "rank[" + std::to_string(h) + "] = " + std::to_string(r) +
                            " is neither SKETCHSSM_DENSE nor in [1, rank_cap]");
        rtot += r;
    }
    if (rtot > (1LL << 30)) return fail(SKETCHSSM_ERR_UNSUPPORTED, "too many sketch rows");

    sketchssm_plan *p = new sketchssm_plan();
    p->d = d;
    p->Hg = H / G;
    p->hpq = H / d.qk_heads;
    p->wait_limit = sk::DEFAULT_WAIT_CYCLES;
    if (!sk::decode_geometry(d.kind, d.value_dim, d.window, d.rank_cap, p->Hg, &p->geo)) {
        delete p;
        return fail(SKETCHSSM_ERR_UNSUPPORTED, "a decode work item of this shape does not fit in shared memory");
    }
    cudaGetDevice(&p->device);
    p->sms = 148;
    cudaDeviceGetAttribute(&p->sms, cudaDevAttrMultiProcessorCount, p->device);
    p->d_rank = p->d_off = p->d_rmax = p->d_coff = p->d_work = p->d_rec = p->d_qk_rneed = nullptr;
    p->d_counts = p->d_status = nullptr;
    p->d_scratch = nullptr;
    cudaStream_t st = (cudaStream_t)stream;
    auto bail = [&](cudaError_t e, const char *what) {
        sketchssm_plan_destroy(p);
        return cuda_fail(e, what);
    };
    const int W = d.window;
    const size_t stride = (size_t)H + G;
    cudaError_t e;
    if ((e = cudaMalloc(&p->d_rank, sizeof(int) * H)) != cudaSuccess) return bail(e, "cudaMalloc");
    if ((e = cudaMalloc(&p->d_off, sizeof(int) * (H + 1))) != cudaSuccess) return bail(e, "cudaMalloc");
    if ((e = cudaMalloc(&p->d_rmax, sizeof(int) * G)) != cudaSuccess) return bail(e, "cudaMalloc");
    if ((e = cudaMalloc(&p->d_coff, sizeof(int) * H)) != cudaSuccess) return bail(e, "cudaMalloc");
    if ((e = cudaMalloc(&p->d_work, sizeof(int) * stride * W)) != cudaSuccess) return bail(e, "cudaMalloc");
    if ((e = cudaMalloc(&p->d_rec, sizeof(int) * 8 * stride * W)) != cudaSuccess) return bail(e, "cudaMalloc");
    if ((e = cudaMalloc(&p->d_qk_rneed, sizeof(int) * d.qk_heads)) != cudaSuccess) return bail(e, "cudaMalloc");
    if ((e = cudaMalloc(&p->d_counts, sizeof(int) * (3 + W))) != cudaSuccess) return bail(e, "cudaMalloc");
    if ((e = cudaMalloc(&p->d_status, sizeof(int))) != cudaSuccess) return bail(e, "cudaMalloc");
    if ((e = cudaMemsetAsync(p->d_status, 0, sizeof(int), st)) != cudaSuccess) return bail(e, "cudaMemsetAsync");
    if ((e = cudaMemcpyAsync(p->d_rank, rank_host, sizeof(int) * H, cudaMemcpyHostToDevice, st)) !=
        cudaSuccess)
        return bail(e, "cudaMemcpyAsync(rank)");
    if ((e = sk::launch_layout(p->d_rank, H, G, d.qk_heads, W, d.rank_cap, p->geo.stage_rows, p->geo.maxnh,
                               p->d_off, p->d_rmax, p->d_coff, p->d_work, p->d_rec, p->d_qk_rneed, p->d_counts,
                               st)) != cudaSuccess)
        return bail(e, "layout kernel launch");
    std::vector<int> counts(3 + W);
    p->h_off.resize(H + 1);
    p->h_rmax.resize(G);
    p->h_work.resize(stride * W);
    if ((e = cudaMemcpyAsync(counts.data(), p->d_counts, sizeof(int) * (3 + W), cudaMemcpyDeviceToHost, st)) !=
            cudaSuccess ||
        (e = cudaMemcpyAsync(p->h_off.data(), p->d_off, sizeof(int) * (H + 1), cudaMemcpyDeviceToHost, st)) !=
            cudaSuccess ||
        (e = cudaMemcpyAsync(p->h_rmax.data(), p->d_rmax, sizeof(int) * G, cudaMemcpyDeviceToHost, st)) !=
            cudaSuccess ||
        (e = cudaMemcpyAsync(p->h_work.data(), p->d_work, sizeof(int) * stride * W, cudaMemcpyDeviceToHost,
                             st)) != cudaSuccess)
        return bail(e, "cudaMemcpyAsync(layout)");
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return bail(e, "layout kernel");
    if (counts[1] != 0) {
        sketchssm_plan_destroy(p);
        return fail(SKETCHSSM_ERR_INVALID_ARG, "layout kernel found an invalid rank");
    }
    p->n_dense = counts[0];
    p->coef_row = counts[2];
    p->h_items.assign(counts.begin() + 3, counts.end());
    {
        // coefficient scratch: the sketch layout, or the dense-read layout, per batch row
        const size_t dense_row = (size_t)H * sk::coef_block(sk::KDIM, W);
        size_t row = (size_t)p->coef_row > dense_row ? (size_t)p->coef_row : dense_row;
        const size_t dots = (size_t)d.qk_heads * sk::dots_row(W, d.rank_cap);
        if (dots > row) row = dots;
        p->scratch_floats = row * (size_t)d.batch;
        if ((e = cudaMalloc(&p->d_scratch, sizeof(float) * p->scratch_floats)) != cudaSuccess)
            return bail(e, "cudaMalloc(coefficient scratch)");
    }
    p->rtot = p->h_off[H];
    p->h_rank.assign(rank_host, rank_host + H);
    if (p->rtot != rtot) {
        sketchssm_plan_destroy(p);
        return fail(SKETCHSSM_ERR_CUDA, "layout kernel disagrees with the host rank sum");
    }
    *out = p;
    return SKETCHSSM_OK;
}

sketchssm_status sketchssm_plan_query(const sketchssm_plan *p, int64_t *r_total, int32_t *offsets_host,
                                      int32_t *rmax_host, int32_t n_tokens, int32_t *work_host,
                                      int32_t *n_work)
{
    g_last_error.clear();
    if (!p) return fail(SKETCHSSM_ERR_INVALID_ARG, "plan is NULL");
    if (r_total) *r_total = p->rtot;
    if (offsets_host) std::memcpy(offsets_host, p->h_off.data(), sizeof(int32_t) * p->h_off.size());
    if (rmax_host) std::memcpy(rmax_host, p->h_rmax.data(), sizeof(int32_t) * p->h_rmax.size());
    if (!work_host && !n_work) return SKETCHSSM_OK;
    const size_t stride = (size_t)p->d.heads + p->d.groups;
    if (n_tokens < 1 || n_tokens > p->d.window)
        return fail(SKETCHSSM_ERR_INVALID_ARG, "n_tokens outside [1, window]");
    const int items = p->h_items[n_tokens - 1];
    if (work_host)
        std::memcpy(work_host, p->h_work.data() + (size_t)(n_tokens - 1) * stride, sizeof(int32_t) * items);
    if (n_work) *n_work = items;
    return SKETCHSSM_OK;
}

sketchssm_status sketchssm_plan_check(const sketchssm_plan *p, sketchssm_stream stream)
{
    g_last_error.clear();
    sketchssm_status s = check_plan(p);
    if (s != SKETCHSSM_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    int flags = 0;
    cudaError_t e;
    if ((e = cudaMemcpyAsync(&flags, p->d_status, sizeof(int), cudaMemcpyDeviceToHost, st)) != cudaSuccess)
        return cuda_fail(e, "cudaMemcpyAsync(status)");
    if ((e = cudaMemsetAsync(p->d_status, 0, sizeof(int), st)) != cudaSuccess)
        return cuda_fail(e, "cudaMemsetAsync(status)");
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "stream");
    if (flags & sk::SK_STATUS_DECODE_TIMEOUT)
        return fail(SKETCHSSM_ERR_TIMEOUT, "a decode CTA waited past the plan's limit for its bulk copies");
    if (flags & sk::SK_STATUS_BAD_ROW)
        return fail(SKETCHSSM_ERR_INVALID_ARG,
                    "a per-row position or token count was out of range; those rows were left unchanged");
    if (flags & sk::SK_STATUS_STEP_TIMEOUT)
        return fail(SKETCHSSM_ERR_TIMEOUT, "a standard-step CTA waited past the plan's limit for its bulk copies");
    if (flags & sk::SK_STATUS_FLUSH_TIMEOUT)
        return fail(SKETCHSSM_ERR_TIMEOUT, "a flush CTA waited past the plan's limit for its bulk copies");
    if (flags & sk::SK_STATUS_PREFILL_TIMEOUT)
        return fail(SKETCHSSM_ERR_TIMEOUT, "a prefill CTA waited past the plan's limit for its tensor-core products");
    return SKETCHSSM_OK;
}

sketchssm_status sketchssm_plan_set_wait_limit(sketchssm_plan *p, int64_t cycles)
{
    g_last_error.clear();
    if (!p) return fail(SKETCHSSM_ERR_INVALID_ARG, "plan is NULL");
    if (cycles < 1) return fail(SKETCHSSM_ERR_INVALID_ARG, "wait limit must be at least 1 cycle");
    p->wait_limit = cycles;
    return SKETCHSSM_OK;
}

sketchssm_status sketchssm_plan_destroy(sketchssm_plan *p)
{
    if (!p) return SKETCHSSM_OK;
    cudaFree(p->d_rank);
    cudaFree(p->d_off);
    cudaFree(p->d_rmax);
    cudaFree(p->d_coff);
    cudaFree(p->d_work);
    cudaFree(p->d_rec);
    cudaFree(p->d_qk_rneed);
    cudaFree(p->d_scratch);
    cudaFree(p->d_counts);
    cudaFree(p->d_status);
    delete p;
    return SKETCHSSM_OK;
}

}  // extern "C"

namespace {

sketchssm_status flush_impl(const sketchssm_plan *p, float *S, const float *omega, const float *kbuf,
                            const float *vbuf, const float *abuf, const float *bbuf, int32_t n_tokens,
                            const int32_t *row_n, float *Y, sketchssm_stream stream)
{
    g_last_error.clear();
    sketchssm_status s = check_plan(p);
    if (s != SKETCHSSM_OK) return s;
    const sketchssm_desc &d = p->d;
    if (n_tokens < 0 || n_tokens > d.window) return fail(SKETCHSSM_ERR_INVALID_ARG, "n_tokens outside [0, window]");
    if (row_n) CHECK_T(row_n, sizeof(int32_t) * (size_t)d.batch, "n_tokens (per row)", false);
    const long long B = d.batch, H = d.heads, Q = d.qk_heads, K = d.key_dim, V = d.value_dim, W = d.window;
    const long long da = d.kind == SKETCHSSM_KDA ? K : 1;
    const bool mamba = d.kind == SKETCHSSM_MAMBA2;
    const bool any_sketch = p->rtot > 0;
    const bool toks = n_tokens > 0;
    CHECK_T(S, fbytes(B, H, K, V), "S", false);
    CHECK_T(omega, any_sketch ? fbytes(d.groups, d.basis_rows, K) : 0, "omega", !any_sketch);
    CHECK_T(Y, any_sketch ? fbytes(B, p->rtot, V) : 0, "Y", !any_sketch);
    CHECK_T(kbuf, toks ? fbytes(B, Q, W, K) : 0, "kbuf", !toks);
    CHECK_T(vbuf, toks ? fbytes(B, H, W, V) : 0, "vbuf", !toks);
    CHECK_T(abuf, toks ? fbytes(B, H, W, da) : 0, "abuf", !toks);
    CHECK_T(bbuf, (toks && !mamba) ? fbytes(B, H, W) : 0, "bbuf", !toks || mamba);
    sk::FlushArgs A;
    A.kind = d.kind;
    A.B = d.batch;
    A.H = d.heads;
    A.Hqk = d.qk_heads;
    A.V = d.value_dim;
    A.W = d.window;
    A.G = d.groups;
    A.Rb = d.basis_rows;
    A.cap = d.rank_cap;
    A.n = n_tokens;
    A.Hg = p->Hg;
    A.hpq = p->hpq;
    A.VS = sk::flush_slab(d.value_dim);
    A.rcap = 0;
    for (int r : p->h_rmax) A.rcap = r > A.rcap ? r : A.rcap;
    A.rmax = p->d_rmax;
    A.status = p->d_status;
    A.wait_limit = p->wait_limit;
    A.row_n = row_n;
    A.rtot = p->rtot;
    A.rank = p->d_rank;
    A.off = p->d_off;
    A.S = S;
    A.omega = omega;
    A.kbuf = kbuf;
    A.vbuf = vbuf;
    A.abuf = abuf;
    A.bbuf = bbuf;
    A.Y = Y;
    cudaError_t e = sk::launch_flush(A, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "flush kernel launch");
    return SKETCHSSM_OK;
}

}  // namespace

extern "C" {

sketchssm_status sketchssm_flush(const sketchssm_plan *p, float *S, const float *omega, const float *kbuf,
                                 const float *vbuf, const float *abuf, const float *bbuf, int32_t n_tokens,
                                 float *Y, sketchssm_stream stream)
{
    return flush_impl(p, S, omega, kbuf, vbuf, abuf, bbuf, n_tokens, nullptr, Y, stream);
}

sketchssm_status sketchssm_flush_rows(const sketchssm_plan *p, float *S, const float *omega, const float *kbuf,
                                      const float *vbuf, const float *abuf, const float *bbuf,
                                      const int32_t *n_tokens, float *Y, sketchssm_stream stream)
{
    g_last_error.clear();
    if (!n_tokens) return fail(SKETCHSSM_ERR_INVALID_ARG, "n_tokens (per row) is NULL");
    return flush_impl(p, S, omega, kbuf, vbuf, abuf, bbuf, p ? p->d.window : 0, n_tokens, Y, stream);
}

sketchssm_status sketchssm_decode_rows(const sketchssm_plan *p, const int32_t *pos, const float *q, const float *k,
                                       const float *v, const float *a, const float *beta, float *kbuf, float *vbuf,
                                       float *abuf, float *bbuf, const float *Y, const float *omega, const float *S,
                                       float *y, sketchssm_stream stream)
{
    g_last_error.clear();
    sketchssm_status s = check_plan(p);
    if (s != SKETCHSSM_OK) return s;
    const sketchssm_desc &d = p->d;
    CHECK_T(pos, sizeof(int32_t) * (size_t)d.batch, "pos (per row)", false);
    if ((s = check_decode_common(p, 0, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, y)) != SKETCHSSM_OK) return s;
    const bool any_sketch = p->rtot > 0, any_dense = p->n_dense > 0;
    CHECK_T(Y, any_sketch ? fbytes(d.batch, p->rtot, d.value_dim) : 0, "Y", !any_sketch);
    CHECK_T(omega, any_sketch ? fbytes(d.groups, d.basis_rows, d.key_dim) : 0, "omega", !any_sketch);
    CHECK_T(S, any_dense ? fbytes(d.batch, d.heads, d.key_dim, d.value_dim) : 0, "S", !any_dense);
    sk::DecodeArgs A = decode_args(p, 0, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, Y, omega, S, y, 0);
    // every row reads its own work list (the launch covers the longest)
    A.row_pos = pos;
    A.work = p->d_work;
    A.rec = p->d_rec;
    int most = 0;
    for (int c : p->h_items) most = c > most ? c : most;
    A.n_items = most;
    cudaError_t e = sk::launch_decode(A, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
    return SKETCHSSM_OK;
}

sketchssm_status sketchssm_decode(const sketchssm_plan *p, int32_t pos, const float *q, const float *k,
                                  const float *v, const float *a, const float *beta, float *kbuf, float *vbuf,
                                  float *abuf, float *bbuf, const float *Y, const float *omega, const float *S,
                                  float *y, sketchssm_stream stream)
{
    g_last_error.clear();
    sketchssm_status s = check_plan(p);
    if (s != SKETCHSSM_OK) return s;
    if ((s = check_decode_common(p, pos, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, y)) != SKETCHSSM_OK)
        return s;
    const sketchssm_desc &d = p->d;
    const bool any_sketch = p->rtot > 0, any_dense = p->n_dense > 0;
    CHECK_T(Y, any_sketch ? fbytes(d.batch, p->rtot, d.value_dim) : 0, "Y", !any_sketch);
    CHECK_T(omega, any_sketch ? fbytes(d.groups, d.basis_rows, d.key_dim) : 0, "omega", !any_sketch);
    CHECK_T(S, any_dense ? fbytes(d.batch, d.heads, d.key_dim, d.value_dim) : 0, "S", !any_dense);
    const sk::DecodeArgs A = decode_args(p, pos, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, Y, omega, S, y, 0);
    cudaError_t e = sk::launch_decode(A, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
    return SKETCHSSM_OK;
}

sketchssm_status sketchssm_dense_decode(const sketchssm_plan *p, int32_t pos, const float *q, const float *k,
                                        const float *v, const float *a, const float *beta, float *kbuf,
                                        float *vbuf, float *abuf, float *bbuf, const float *S, float *y,
                                        sketchssm_stream stream)
{
    g_last_error.clear();
    sketchssm_status s = check_plan(p);
    if (s != SKETCHSSM_OK) return s;
    if ((s = check_decode_common(p, pos, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, y)) != SKETCHSSM_OK)
        return s;
    const sketchssm_desc &d = p->d;
    CHECK_T(S, fbytes(d.batch, d.heads, d.key_dim, d.value_dim), "S", false);
    const sk::DecodeArgs A = decode_args(p, pos, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, nullptr, nullptr, S, y, 1);
    cudaError_t e = sk::launch_decode(A, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "dense decode kernel launch");
    return SKETCHSSM_OK;
}

}  // extern "C"

// ============================================================================ static scratch
//
// sketchssm_decode_static_scratch: the sketch decode with its scratch in a file-scope
// static device array instead of the plan's cudaMalloc'd buffer.  It serves callers
// that must not allocate device memory once serving has started (an engine whose HBM
// is fully committed to its own state / KV pools, where a cudaMalloc would fail or
// make the pool release memory, and code that cannot take the device-wide
// synchronisation cudaMalloc / cudaFree may imply).  Nothing below allocates.
//
// The array is shared by every call on a device; calls that overlap on the GPU race
// on it.  Nothing in it needs to start at zero: the products kernel writes every
// entry the combine kernel reads before the combine reads it.

static __device__ __align__(256) float g_static_scratch[SKETCHSSM_STATIC_SCRATCH_BYTES / sizeof(float)];

namespace {

// The array's address on the current device.  Looked up on every call: the lookup
// allocates nothing, and a cached address would go stale if the device's context were
// destroyed and created again (cudaDeviceReset), which reloads the library's device code.
// The first lookup on a device may load that code there.
sketchssm_status static_scratch(float **out)
{
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    *out = static_cast<float *>(p);
    return SKETCHSSM_OK;
}

// floats of scratch the sketch decode of plan p reads and writes
size_t sketch_scratch_floats(const sketchssm_plan *p)
{
    const sketchssm_desc &d = p->d;
    const size_t per_row = d.kind == SKETCHSSM_MAMBA2 ? (size_t)d.qk_heads * sk::dots_row(d.window, d.rank_cap)
                                                      : (size_t)p->coef_row;
    return per_row * (size_t)d.batch;
}

}  // namespace

extern "C" sketchssm_status sketchssm_decode_static_scratch(const sketchssm_plan *p, int32_t pos, const float *q,
                                                            const float *k, const float *v, const float *a,
                                                            const float *beta, float *kbuf, float *vbuf,
                                                            float *abuf, float *bbuf, const float *Y,
                                                            const float *omega, const float *S, float *y,
                                                            sketchssm_stream stream)
{
    g_last_error.clear();
    sketchssm_status s = check_plan(p);
    if (s != SKETCHSSM_OK) return s;
    const size_t need = sketch_scratch_floats(p) * sizeof(float);
    if (need > SKETCHSSM_STATIC_SCRATCH_BYTES)
        return fail(SKETCHSSM_ERR_INVALID_ARG, "static scratch: this plan's decode needs " + std::to_string(need) +
                                                   " bytes, the static array holds " +
                                                   std::to_string(SKETCHSSM_STATIC_SCRATCH_BYTES) +
                                                   " (use sketchssm_decode)");
    if ((s = check_decode_common(p, pos, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, y)) != SKETCHSSM_OK)
        return s;
    const sketchssm_desc &d = p->d;
    const bool any_sketch = p->rtot > 0, any_dense = p->n_dense > 0;
    CHECK_T(Y, any_sketch ? fbytes(d.batch, p->rtot, d.value_dim) : 0, "Y", !any_sketch);
    CHECK_T(omega, any_sketch ? fbytes(d.groups, d.basis_rows, d.key_dim) : 0, "omega", !any_sketch);
    CHECK_T(S, any_dense ? fbytes(d.batch, d.heads, d.key_dim, d.value_dim) : 0, "S", !any_dense);
    float *scratch = nullptr;
    if ((s = static_scratch(&scratch)) != SKETCHSSM_OK) return s;
    sk::DecodeArgs A = decode_args(p, pos, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, Y, omega, S, y, 0);
    A.scratch = scratch;
    cudaError_t e = sk::launch_decode(A, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch (static scratch)");
    return SKETCHSSM_OK;
}

extern "C" sketchssm_status sketchssm_prefill(const sketchssm_plan *p, int32_t T, const float *k, const float *v,
                                              const float *a, const float *beta, float *S, const float *omega,
                                              float *Y, sketchssm_stream stream)
{
    g_last_error.clear();
    sketchssm_status s = check_plan(p);
    if (s != SKETCHSSM_OK) return s;
    if (T < 0) return fail(SKETCHSSM_ERR_INVALID_ARG, "T < 0");
    const sketchssm_desc &d = p->d;
    const long long B = d.batch, H = d.heads, Q = d.qk_heads, K = d.key_dim, V = d.value_dim;
    const long long da = d.kind == SKETCHSSM_KDA ? K : 1;
    const bool mamba = d.kind == SKETCHSSM_MAMBA2;
    const bool toks = T > 0;
    if ((long long)B * H * (V / sk::step_slab(d.value_dim)) > 0x7fffffffLL)
        return fail(SKETCHSSM_ERR_UNSUPPORTED, "batch * heads too large for one prefill launch");
    CHECK_T(k, toks ? fbytes(B, T, Q, K) : 0, "k", !toks);
    CHECK_T(v, toks ? fbytes(B, T, H, V) : 0, "v", !toks);
    CHECK_T(a, toks ? fbytes(B, T, H, da) : 0, "a", !toks);
    CHECK_T(beta, (toks && !mamba) ? fbytes(B, T, H) : 0, "beta", !toks || mamba);
    CHECK_T(S, fbytes(B, H, K, V), "S", false);
    // the sketch's tensors too, before S is touched (the flush below checks them again)
    const bool any_sketch = p->rtot > 0;
    CHECK_T(omega, any_sketch ? fbytes(d.groups, d.basis_rows, K) : 0, "omega", !any_sketch);
    CHECK_T(Y, any_sketch ? fbytes(B, p->rtot, V) : 0, "Y", !any_sketch);
    if (toks) {
        sk::PrefillArgs A;
        A.kind = d.kind;
        A.B = d.batch;
        A.H = d.heads;
        A.Hqk = d.qk_heads;
        A.V = d.value_dim;
        A.hpq = p->hpq;
        A.T = T;
        A.VS = sk::step_slab(d.value_dim);
        A.k = k;
        A.v = v;
        A.a = a;
        A.beta = beta;
        A.S = S;
        A.status = p->d_status;
        A.wait_limit = p->wait_limit;
        cudaError_t e = sk::launch_prefill(A, (cudaStream_t)stream);
        if (e != cudaSuccess) return cuda_fail(e, "prefill kernel launch");
    }
    // the handoff: the sketch of the new state (no buffered tokens)
    return flush_impl(p, S, omega, nullptr, nullptr, nullptr, nullptr, 0, nullptr, Y, stream);
}

extern "C" sketchssm_status sketchssm_step(const sketchssm_plan *p, const float *q, const float *k,
                                           const float *v, const float *a, const float *beta, float *S,
                                           float *y, sketchssm_stream stream)
{
    g_last_error.clear();
    sketchssm_status s = check_plan(p);
    if (s != SKETCHSSM_OK) return s;
    const sketchssm_desc &d = p->d;
    const long long B = d.batch, H = d.heads, Q = d.qk_heads, K = d.key_dim, V = d.value_dim;
    const long long da = d.kind == SKETCHSSM_KDA ? K : 1;
    const bool mamba = d.kind == SKETCHSSM_MAMBA2;
    CHECK_T(q, fbytes(B, Q, K), "q", false);
    CHECK_T(k, fbytes(B, Q, K), "k", false);
    CHECK_T(v, fbytes(B, H, V), "v", false);
    CHECK_T(a, fbytes(B, H, da), "a", false);
    CHECK_T(beta, mamba ? 0 : fbytes(B, H), "beta", mamba);
    CHECK_T(S, fbytes(B, H, K, V), "S", false);
    CHECK_T(y, fbytes(B, H, V), "y", false);
    sk::StepArgs A;
    A.kind = d.kind;
    A.B = d.batch;
    A.H = d.heads;
    A.Hqk = d.qk_heads;
    A.V = d.value_dim;
    A.hpq = p->hpq;
    A.VS = sk::step_slab(d.value_dim);
    A.wait_limit = p->wait_limit;
    A.status = p->d_status;
    A.q = q;
    A.k = k;
    A.v = v;
    A.a = a;
    A.beta = beta;
    A.S = S;
    A.y = y;
    cudaError_t e = sk::launch_step(A, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "standard step kernel launch");
    return SKETCHSSM_OK;
}
