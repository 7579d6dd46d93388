/*
 * sketchssm.h -- C ABI of the B200 (sm_100a) SketchSSM decode path.
 *
 * SketchSSM ("SketchSSM: Write to the Full State, Read from a Compact Sketch",
 * paper abstract on the newx.sg and mlsanity pages) keeps the full fp32 recurrent
 * state S (K x V per state head) up to date, but reads it only at state updates.
 * Keys and values are buffered for a window of W tokens (ReplaySSM).  At each
 * update (a "flush") the buffered tokens are applied to S and the new S is read
 * once to form, for every sketch head, the r x V sketch Y = Omega_r S, Omega_r being
 * the first r rows of the head group's fixed orthonormal basis.  Every decode step
 * then forms the coefficients c = Omega_r q0 and returns
 *     y = Y^T c + (exact replay of the buffered tokens),
 * never touching S.  Heads allotted no rank ("dense fallback", sketchssm PyPI page,
 * calibration stage "allocate") read S exactly.
 *
 * Recurrences (per state head, token i with key k_i, value v_i):
 *     S <- M_i S + beta_i k_i v_i^T
 *     Mamba-2 : M_i = a_i I,                        beta_i = 1   (a_i scalar)
 *     GDN     : M_i = a_i (I - beta_i k_i k_i^T)                 (a_i scalar)
 *     KDA     : M_i = diag(a_i) (I - beta_i k_i k_i^T)           (a_i in R^K)
 * The output of a step is read after its own token is applied: y_t = S_t^T q_t.
 *
 * General conventions (every call):
 *  - All tensors are fp32, C-contiguous, device memory owned by the caller, and
 *    16-byte aligned (else SKETCHSSM_ERR_ALIGNMENT).  A pointer that is not device
 *    accessible (plain host memory) is rejected with SKETCHSSM_ERR_INVALID_ARG.
 *  - Layouts (B batch rows, H state heads, Hqk q/k heads, G basis groups, Rb basis
 *    rows per group, W window, Rtot = sum of the sketch heads' ranks):
 *        S     [B][H][K][V]         omega [G][Rb][K]       Y   [B][Rtot][V]
 *        q, k  [B][Hqk][K]          v     [B][H][V]        y   [B][H][V]
 *        a     [B][H]   (KDA [B][H][K])                    beta [B][H]
 *        kbuf  [B][Hqk][W][K]       vbuf  [B][H][W][V]
 *        abuf  [B][H][W] (KDA [B][H][W][K])                bbuf [B][H][W]
 *    Head h belongs to basis group h / (H/G) and uses q/k head h / (H/Hqk).
 *    Sketch head h owns rows off[h] .. off[h]+rank[h]-1 of Y (off = exclusive
 *    prefix sum of the sketch ranks in head order; dense heads own no rows).
 *  - beta and bbuf are ignored for Mamba-2 and may be NULL there.
 *  - Every call is asynchronous and stream ordered (stream = a cudaStream_t, NULL
 *    for the legacy default stream).  Arguments are checked on the host before any
 *    launch; a call that returns an error launched nothing and wrote nothing.  A
 *    failed launch returns SKETCHSSM_ERR_CUDA; sketchssm_last_error() then gives
 *    the CUDA error text.  No call allocates or frees caller memory.  No kernel
 *    waits on another CTA; a decode or flush CTA waits, with a bound, only for its
 *    own bulk copies, and records a timeout that sketchssm_plan_check reports.
 *  - Decode / flush protocol: pos counts the tokens buffered since the last flush.
 *    sketchssm_decode(pos) appends the step's token at buffer slot pos and returns
 *    y including it.  After the decode at pos = W-1 the caller runs
 *    sketchssm_flush(n_tokens = W) and restarts at pos = 0.  sketchssm_flush with
 *    n_tokens = 0 forms the sketch of an initial state; sketchssm_prefill applies a
 *    prompt to the state and then forms its sketch, after which decoding starts at
 *    pos = 0.
 *  - Supported shapes: K = 128, V a multiple of 16 in [16, 256], 1 <= W <= 32,
 *    H divisible by G with H/G <= 32, Hqk dividing H and divisible by G,
 *    1 <= rank_cap <= basis_rows <= K.  Others return SKETCHSSM_ERR_UNSUPPORTED.
 *  - Calls on one plan from several host threads are safe; calls whose kernels
 *    overlap on the GPU and write the same buffers race, as with any kernel.
 */
#ifndef SKETCHSSM_H
#define SKETCHSSM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SKETCHSSM_OK = 0,
    SKETCHSSM_ERR_INVALID_ARG = 1,  /* bad pointer, size, rank value or descriptor */
    SKETCHSSM_ERR_ALIGNMENT = 2,    /* a tensor pointer is not 16-byte aligned */
    SKETCHSSM_ERR_UNSUPPORTED = 3,  /* valid, but outside the shapes built for */
    SKETCHSSM_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    SKETCHSSM_ERR_TIMEOUT = 5       /* a kernel wait ran past its limit (sketchssm_plan_check) */
} sketchssm_status;

typedef enum {
    SKETCHSSM_MAMBA2 = 0,  /* scalar decay per head ("Transformers are SSMs") */
    SKETCHSSM_GDN = 1,     /* gated delta rule ("Gated Delta Networks") */
    SKETCHSSM_KDA = 2      /* per-key-channel decay with the delta rule */
} sketchssm_kind;

/* rank-table value of a dense-fallback head (PyPI page, stage "allocate") */
#define SKETCHSSM_DENSE (-1)

/* Shape of one recurrent layer at a fixed batch. */
typedef struct {
    int32_t kind;        /* sketchssm_kind */
    int32_t batch;       /* B >= 1 */
    int32_t heads;       /* H: state heads */
    int32_t qk_heads;    /* Hqk: heads carrying q and k (G for Mamba-2 groups, H per head) */
    int32_t key_dim;     /* K (128 on the Nemotron Nano calibration card) */
    int32_t value_dim;   /* V (80 on the card) */
    int32_t window;      /* W (16 on the card) */
    int32_t groups;      /* G: basis groups (8 on the card), contiguous runs of H/G heads */
    int32_t basis_rows;  /* Rb: rows stored per group basis (79 on the card) */
    int32_t rank_cap;    /* largest allowed rank (49 on the card) */
} sketchssm_desc;

/* Opaque plan: the layer's shape plus its device-side rank / offset / work tables. */
typedef struct sketchssm_plan sketchssm_plan;

/* A cudaStream_t, passed as a plain pointer. */
typedef void *sketchssm_stream;

/*
 * Create a plan: checks desc, copies the per-head rank table (host, [H] int32,
 * values SKETCHSSM_DENSE or 1..rank_cap) to the device and runs the layout kernel,
 * which computes the packed sketch offsets off[H+1], the largest rank per group
 * rmax[G] and, for every number n = 1..W of replayed tokens, the CTA work list of
 * one batch row of the decode launch: one item per dense head in head order, then
 * per group its sketch heads packed greedily in head order into items whose rows
 * (rank + n per head) fit one shared-memory stage.  The plan owns those device
 * tables (freed by sketchssm_plan_destroy).  Synchronises `stream` once, so that
 * the host knows Rtot and the item counts.  *out is set only on success.
 * Source: the calibration stage "allocate" of the sketchssm PyPI page (each head
 * gets a rank or falls back to dense) and its stage "basis" (one basis per group).
 *
 * group_host: the basis group of every head (host, [H] int32, values 0..G-1), or NULL
 * for the layout the kernels are built for: contiguous runs of H/G heads, head h in
 * group h / (H/G) (Mamba-2's heads of one B/C group sit side by side).  A table equal to
 * that layout is accepted; any other map returns SKETCHSSM_ERR_UNSUPPORTED (a value
 * outside 0..G-1: SKETCHSSM_ERR_INVALID_ARG).  Heads are independent on this path, so a
 * caller whose groups interleave numbers its heads group by group (permuting the head
 * axis of its q/k/v/a/beta/S tensors and the rank table alike) and gets the same result.
 */
sketchssm_status sketchssm_plan_create(const sketchssm_desc *desc, const int32_t *rank_host,
                                       const int32_t *group_host, sketchssm_stream stream,
                                       sketchssm_plan **out);

/*
 * Copy the plan's layout tables to host memory (reads host copies; no GPU work).
 * Any output pointer may be NULL.  offsets_host gets H+1 values, rmax_host G
 * values, *r_total Rtot (the number of sketch rows of Y), and work_host the work
 * list for n_tokens (1..W) replayed tokens, at most G+H entries, *n_work their
 * count.  Entry < 0: dense item for head -entry-1; entry >= 0: sketch item holding
 * the sketch heads among heads entry/64 .. entry/64 + entry%64 - 1.
 */
sketchssm_status sketchssm_plan_query(const sketchssm_plan *plan, int64_t *r_total,
                                      int32_t *offsets_host, int32_t *rmax_host, int32_t n_tokens,
                                      int32_t *work_host, int32_t *n_work);

/*
 * Synchronise `stream`, then report what the kernels recorded on the plan since the
 * last check, and clear it: SKETCHSSM_ERR_TIMEOUT if a decode, flush, standard-step or
 * prefill CTA waited longer than the plan's wait limit (sketchssm_plan_set_wait_limit;
 * default about a second) for its own bulk copies (the Mamba-2 prefill: for its own
 * tensor-core products); SKETCHSSM_OK otherwise.  Such a CTA records the timeout and
 * keeps waiting, up to the default limit more, for the same operations, so the outputs
 * are complete unless that second wait also ran out (then the CTA gives up and its
 * outputs are incomplete).  No kernel waits on anything but its own operations, so a
 * timeout at the default limit means a fault of the copy engine or the tensor core, not
 * a deadlock.
 */
sketchssm_status sketchssm_plan_check(const sketchssm_plan *plan, sketchssm_stream stream);

/*
 * Set the plan's wait limit: the SM clock cycles (>= 1; default 2e9, about a second)
 * a CTA waits for its own bulk copies before it records a timeout.  A diagnostic and
 * a test hook: with a limit of a few cycles most waits run past it, and
 * sketchssm_plan_check reports SKETCHSSM_ERR_TIMEOUT while the results stay complete.
 * Applies to calls made after it; must not race with other calls on the plan.
 */
sketchssm_status sketchssm_plan_set_wait_limit(sketchssm_plan *plan, int64_t cycles);

/* Free a plan and its device tables.  NULL is accepted.  Must not race with calls
 * that use the plan; device work already queued keeps its own copy of nothing, so
 * synchronise the streams that used the plan first. */
sketchssm_status sketchssm_plan_destroy(sketchssm_plan *plan);

/*
 * Flush (write-full step; paper abstract: updates always reach the full state, which
 * is read only here, once, to compute the basis outputs kept as the sketch).  For
 * every (b, h) apply buffer slots 0..n_tokens-1 in
 * order to S (in place), then write Y rows of every sketch head:
 *     Y[b][off[h] + m][:] = sum_k omega[g(h)][m][k] S[b][h][k][:],  m < rank[h].
 * n_tokens in [0, W]; with 0, S is left untouched and only Y is formed.
 * Reads kbuf, vbuf, abuf, bbuf (slots < n_tokens), omega.  Writes S (if
 * n_tokens > 0) and Y.  Y may be NULL only if the plan has no sketch head.
 */
sketchssm_status sketchssm_flush(const sketchssm_plan *plan, float *S, const float *omega,
                                 const float *kbuf, const float *vbuf, const float *abuf,
                                 const float *bbuf, int32_t n_tokens, float *Y,
                                 sketchssm_stream stream);

/*
 * Sketch decode (read-sketch step; SketchSSM, Abstract: the output of a decode step is
 * rebuilt from the sketch rows weighted by coefficients taken from the query, and the
 * full state is not read).  pos in [0, W): tokens buffered since the last flush.  Appends the step's
 * token (k, v, a, beta) at buffer slot pos, then for every (b, h) with n = pos+1:
 *   replay: walk the buffered tokens newest first with x = q,
 *           y += beta_i (k_i . x) v_i,  x <- M_i^T x;      q0 = final x
 *           (Mamba-2: y = sum_i w_i (k_i . q) v_i, w_i = prod_{j>i} a_j,
 *            q0 = (prod_j a_j) q)
 *   read:   sketch head: c = Omega_r q0, y += Y_h^T c;   dense head: y += S_h^T q0.
 * Reads q, k, v, a, beta, the buffers' slots < pos, Y, omega and (dense heads
 * only) S.  Writes y and buffer slot pos.  Y / omega may be NULL only if the plan
 * has no sketch head; S may be NULL only if it has no dense head.
 */
sketchssm_status sketchssm_decode(const sketchssm_plan *plan, int32_t pos, const float *q,
                                  const float *k, const float *v, const float *a,
                                  const float *beta, float *kbuf, float *vbuf, float *abuf,
                                  float *bbuf, const float *Y, const float *omega,
                                  const float *S, float *y, sketchssm_stream stream);

/*
 * Dense-read decode: the ReplaySSM baseline the paper improves on (SketchSSM, Abstract:
 * with buffered updates alone, every query still reads the whole state).  Same as
 * sketchssm_decode, but every head
 * reads S exactly (y += S_h^T q0) whatever its rank.  Reads S, never Y or omega.
 */
sketchssm_status sketchssm_dense_decode(const sketchssm_plan *plan, int32_t pos, const float *q,
                                        const float *k, const float *v, const float *a,
                                        const float *beta, float *kbuf, float *vbuf,
                                        float *abuf, float *bbuf, const float *S, float *y,
                                        sketchssm_stream stream);

/*
 * Sketch decode whose scratch comes from a fixed static device array instead of the
 * plan's buffer; the paper has no counterpart (it is a memory-ownership variant of
 * sketchssm_decode, with the same arguments and layouts).  It runs the two-launch form
 * of the decode (products, then combine), whose products pass through scratch; its
 * results equal sketchssm_decode's up to fp32 rounding (for Mamba-2, sketchssm_decode
 * runs the one-launch form, which sums the same terms in another order).
 *
 * For callers that must not allocate device memory at all once serving has started:
 * an engine that has handed every free byte of HBM to its own state and KV pools, so
 * that a cudaMalloc would fail or force its pool to give memory back, and code that
 * cannot afford the device-wide synchronisation cudaMalloc / cudaFree may imply.
 * This call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine): the coefficient / product rows live in one array of
 * SKETCHSSM_STATIC_SCRATCH_BYTES per device, linked into the library.
 *  - Limit: a plan whose sketch decode needs more than SKETCHSSM_STATIC_SCRATCH_BYTES
 *    (Mamba-2: batch * qk_heads * round4(window + rank_cap) floats; GDN / KDA: batch
 *    * the plan's coefficient floats per batch row) returns SKETCHSSM_ERR_INVALID_ARG
 *    with the sizes in sketchssm_last_error(), before any tensor is looked at.
 *  - Set-up: every call looks the array's address up on the current device (the plan
 *    check already requires the plan's device to be current); the lookup allocates
 *    nothing.  The first lookup on a device may load the library's device code there,
 *    so make the first call on each device before any stream capture.
 *  - Sharing: every call on a device, from every plan and host thread, uses the same
 *    array.  Calls whose kernels overlap on the GPU (different streams without an
 *    ordering between them) race on it and give wrong results; calls in stream order
 *    do not.
 *  - Nothing in the array needs to start at zero: each call writes every scratch entry
 *    it reads before reading it, so stale contents of an earlier call do not matter.
 */
#define SKETCHSSM_STATIC_SCRATCH_BYTES (8u << 20)

sketchssm_status sketchssm_decode_static_scratch(const sketchssm_plan *plan, int32_t pos,
                                                 const float *q, const float *k, const float *v,
                                                 const float *a, const float *beta, float *kbuf,
                                                 float *vbuf, float *abuf, float *bbuf,
                                                 const float *Y, const float *omega,
                                                 const float *S, float *y,
                                                 sketchssm_stream stream);

/*
 * Per-sequence positions (continuous batching): sketchssm_decode with a position per
 * batch row.  pos is a device array [B] of int32 (16-byte aligned); row b appends its
 * token at its own buffer slot pos[b] and replays pos[b] + 1 tokens.  Rows move through
 * their windows independently; sketchssm_flush_rows applies each row's tokens.  A
 * position outside [0, W) cannot be seen on the host: the kernels leave that row
 * unchanged (no y, no append) and sketchssm_plan_check reports SKETCHSSM_ERR_INVALID_ARG.
 * Everything else as sketchssm_decode.  Source: the serving setting of the sketchssm
 * PyPI page (vLLM batches sequences at different positions).
 */
sketchssm_status sketchssm_decode_rows(const sketchssm_plan *plan, const int32_t *pos, const float *q,
                                       const float *k, const float *v, const float *a,
                                       const float *beta, float *kbuf, float *vbuf, float *abuf,
                                       float *bbuf, const float *Y, const float *omega,
                                       const float *S, float *y, sketchssm_stream stream);

/*
 * Per-row flush: sketchssm_flush with a token count per batch row.  n_tokens is a device
 * array [B] of int32 in [0, W] (16-byte aligned); row b applies its buffer slots
 * 0 .. n_tokens[b]-1 to its state and re-forms its sketch rows.  A row with 0 tokens is
 * left untouched (its state and sketch keep their values; the initial sketch of a fresh
 * state is formed with sketchssm_flush(n_tokens = 0)).  A count outside [0, W] leaves
 * the row untouched and is reported by sketchssm_plan_check as SKETCHSSM_ERR_INVALID_ARG.
 */
sketchssm_status sketchssm_flush_rows(const sketchssm_plan *plan, float *S, const float *omega,
                                      const float *kbuf, const float *vbuf, const float *abuf,
                                      const float *bbuf, const int32_t *n_tokens, float *Y,
                                      sketchssm_stream stream);

/*
 * Standard per-step recurrent decode: the baseline the paper compares against (paper
 * abstract: standard decoding reads and updates the full state for every token).  For
 * every (b, h) apply the step's token to S in place, S <- M S + beta k v^T, and write
 * y[b][h] = S^T q, read after the update.  No buffer or sketch is read or written; the
 * plan supplies only the shape (its rank table is not used).  Tensors and layouts as in
 * the general conventions (q, k [B][Hqk][K], v [B][H][V], a [B][H] or KDA [B][H][K],
 * beta [B][H] or NULL for Mamba-2, S [B][H][K][V], y [B][H][V]).  A state driven only by
 * this call matches the state of the sketch path's decode / flush protocol after every
 * flush (the same recurrence), and y equals the exact read at every step.
 */
sketchssm_status sketchssm_step(const sketchssm_plan *plan, const float *q, const float *k,
                                const float *v, const float *a, const float *beta, float *S,
                                float *y, sketchssm_stream stream);

/*
 * Prefill handoff: the step before decoding.  For every (b, h) the prompt's T tokens
 * are applied to S in place, in order t = 0 .. T-1, with the decode path's recurrence
 * S <- M_t S + beta_t k_t v_t^T (paper abstract: every state update reaches the full
 * state; the pages leave the prompt to the model, so the tokens are applied one after
 * another).  Then Y is formed from the new state exactly as
 * sketchssm_flush(n_tokens = 0) forms it.  The window buffer is not read or written:
 * decoding continues at pos = 0.  T = 0 only forms Y.
 *  - Prompt layouts (token-major, as a model produces them; 16-byte aligned):
 *    k [B][T][Hqk][K], v [B][T][H][V], a [B][T][H] (KDA [B][T][H][K]),
 *    beta [B][T][H] (NULL for Mamba-2).  k, v, a may be NULL when T = 0.
 *  - S [B][H][K][V] is read and written once whatever T; omega and Y as for
 *    sketchssm_flush.
 *  - Mamba-2 prompts of at most 64 tokens with V <= 128 run on the tensor cores
 *    (tcgen05, fp32 accuracy by a three-product tf32 split); other prompts and kinds
 *    apply the tokens in 16-token chunks.
 *  - T < 0 returns SKETCHSSM_ERR_INVALID_ARG; nothing is launched on an error.
 */
sketchssm_status sketchssm_prefill(const sketchssm_plan *plan, int32_t T, const float *k, const float *v,
                                   const float *a, const float *beta, float *S, const float *omega,
                                   float *Y, sketchssm_stream stream);

/* Static text of a status code. */
const char *sketchssm_status_string(sketchssm_status status);

/* Detail of the last error returned on the calling host thread ("" if none). */
const char *sketchssm_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SKETCHSSM_H */
