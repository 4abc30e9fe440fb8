/*
 * lizard.h -- C ABI of the B200 (sm_100a) hybrid attention library.
 *
 * The operator is the hybrid attention of "Lizard: An Efficient Linearization
 * Framework for Large Language Models" (gist.science technical summary,
 * section 2a "hybrid attention architecture"):
 *
 *   gated linear attention   S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T,
 *                            o_gla_t = q_t^T S_t            (state update eq.)
 *   anchor window softmax    o_swa_t = softmax over keys j in [t-w+1, t] plus
 *                            M learnable meta tokens that sit in the
 *                            denominator as attention sinks
 *   output                   o_t = o_gla_t + alpha * o_swa_t  (weighted sum)
 *
 * and the gradient needed by its first training stage (section 2b), plus the
 * constant-memory generation step that the fixed-size state allows.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer is DEVICE memory owned by the caller.  The library never
 *   allocates device memory, frees or synchronizes; every call is
 *   asynchronous on `stream` (a cudaStream_t passed as void*; NULL means the
 *   legacy default stream).  The one resource it creates itself is a
 *   high-priority side stream with two events per (host thread, device),
 *   made on the first lz_hybrid_bwd call and kept: see lz_hybrid_bwd.
 * - Layouts are contiguous row-major:
 *     q, k, g, dq, dk, dg     [B, H, T, dk]
 *     v, o, o_swa, dO, dv     [B, H, T, dv]
 *     h0, hT, dh0, dhT        [B, H, dk, dv]   (fp32)
 *     lse                     [B, H, T]        (fp32, natural log)
 *     meta_k, dmeta_k         [H, M, dk]
 *     meta_v, dmeta_v         [H, M, dv]
 *   q, k, v, o, o_swa, meta_k, meta_v, dO, dq, dk, dv use the I/O dtype
 *   `io`; the log-gates g, states, lse and every meta gradient are fp32.
 * - g holds log-gates (g <= 0; gate = exp(g) in (0, 1]).  g > 0 is not
 *   checked: it is a precondition, and NaN/Inf propagate.
 * - Every pointer must be 16-byte aligned.  Supported: dk, dv in {64, 128};
 *   chunk in {64, 128} (a tiling choice: results agree up to rounding);
 *   1 <= w <= 1024; 0 <= M <= 16; T >= 0 (no multiple-of-anything rule).
 * - Inputs must not alias outputs (the decode state/rings/pos are the
 *   in-place exceptions).  Gradients are written, not accumulated.
 * - On a bad argument the call returns LZ_ERR_INVALID_ARG or
 *   LZ_ERR_UNSUPPORTED before launching anything; a failed launch returns
 *   LZ_ERR_CUDA.  lz_last_error() then describes the failure (thread-local).
 *   Kernels never trap.
 */
#ifndef LIZARD_H
#define LIZARD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LZ_OK = 0,
  LZ_ERR_INVALID_ARG = 1,  /* NULL / misaligned pointer, bad size, short workspace */
  LZ_ERR_UNSUPPORTED = 2,  /* valid but outside the supported shapes/dtypes */
  LZ_ERR_CUDA = 3,         /* a kernel launch or CUDA runtime call failed */
  LZ_ERR_TIMEOUT = 4       /* a bounded device-side wait gave up */
} lz_status;

typedef enum { LZ_F32 = 0, LZ_BF16 = 1 } lz_dtype;

typedef void* lz_stream; /* cudaStream_t */

/* Problem description shared by the prefill/training entry points. */
typedef struct {
  int B, H, T;    /* batch, heads, sequence length */
  int dk, dv;     /* key and value head dims */
  int chunk;      /* chunk length of the gated branch (64 or 128) */
  int w;          /* window: keys t-w+1 .. t (w keys, the current one included) */
  int M;          /* number of meta-memory tokens (0 = none) */
  lz_dtype io;    /* dtype of q, k, v, o, meta, dO, dq, dk, dv */
  float scale;    /* softmax logit scale (usually 1/sqrt(dk)); meta logits too */
  float alpha;    /* weight of the window branch in the hybrid sum */
  int gate_logits;   /* 0: `g` holds fp32 log-gates.  1: `g` holds the gate
                      * LOGITS z, bf16 [B,H,T,dk] (section 2a: the gate is
                      * sigma(W_gamma x), z = W_gamma x); the log-gate is
                      * gate_scale * log sigma(z) (mapped once into the call's
                      * scratch, or inside the kernels: lz_fused_gate_logits),
                      * and the backward's dg receives dL/dz (fp32).  Needs
                      * io = LZ_BF16 and dk = dv = 128 (LZ_ERR_UNSUPPORTED
                      * otherwise).  Zero-initialised dims keep mode 0. */
  float gate_scale;  /* > 0, used when gate_logits = 1 (a temperature; 1 is
                      * the page's gate) */
} lz_dims;

/* Bytes of scratch the call needs (0 is possible); `which` is one of the
 * LZ_WS_* values.  The scratch is caller-owned device memory, 256-byte
 * aligned, and may be reused once the call's stream work has finished.
 * LZ_WS_CHUNK_STATES is not scratch but the size of the optional
 * `chunk_states` buffer of the gated forward and backward calls: the state
 * before every 64-token chunk, [B, H, ceil(T/64), dk, dv] bf16, kept by the
 * forward so that the backward need not walk the sequence again.  It is 0
 * where the kernels keep no such states (fp32 I/O, d = 64); the pointers
 * are then ignored.  With gate_logits = 1 the gated and hybrid scratch also
 * holds B*H*T*dk floats for the mapped log-gates. */
enum { LZ_WS_GLA_FWD = 0, LZ_WS_HYBRID_FWD = 1, LZ_WS_GLA_BWD = 2,
       LZ_WS_SWA_BWD = 3, LZ_WS_HYBRID_BWD = 4, LZ_WS_CHUNK_STATES = 5,
       LZ_WS_HYBRID_FWD_MSE = 6 };
size_t lz_workspace_bytes(const lz_dims* d, int which);

/* Gated linear attention forward (section 2a, state update equation).
 *   o = q^T S_t per token; h0 (nullable = zeros) is the state before token 0;
 *   hT (nullable) receives the state after the last token; chunk_states
 *   (nullable) receives the state before every 64-token chunk (see
 *   LZ_WS_CHUNK_STATES) for lz_gla_bwd.  Fields used: B, H, T, dk, dv,
 *   chunk, io. */
lz_status lz_gla_fwd(const lz_dims* d, const void* q, const void* k,
                     const void* v, const float* g, const float* h0, void* o,
                     float* hT, void* chunk_states, void* ws, size_t ws_bytes,
                     lz_stream stream);

/* Sliding-window softmax with meta-memory sinks (section 2a, anchor window
 * attention).  meta_k may be NULL only when M == 0.  meta_v == NULL selects
 * the sink-only reading (meta tokens enter the denominator only).  o gets
 * o_swa; lse (nullable) gets log(sum of exp(logits)) per query, which the
 * backward needs.  Fields used: B, H, T, dk, dv, w, M, io, scale. */
lz_status lz_swa_meta_fwd(const lz_dims* d, const void* q, const void* k,
                          const void* v, const void* meta_k,
                          const void* meta_v, void* o, float* lse,
                          lz_stream stream);

/* Hybrid forward o = o_gla + alpha * o_swa (section 2a, final output).
 *   hT, lse, o_swa, chunk_states are nullable extra outputs (lse is what
 *   lz_hybrid_bwd needs; o_swa and chunk_states let it skip work).  All
 *   lz_dims fields are used. */
lz_status lz_hybrid_fwd(const lz_dims* d, const void* q, const void* k,
                        const void* v, const float* g, const void* meta_k,
                        const void* meta_v, const float* h0, void* o,
                        float* hT, float* lse, void* o_swa, void* chunk_states,
                        void* ws, size_t ws_bytes, lz_stream stream);

/* lz_hybrid_fwd followed by the first training stage's loss (section 2b,
 * training strategy: the hybrid attention learns to reproduce the teacher's
 * attention output under a mean-squared-error loss).
 *   target: the teacher's output, [B, H, T, dv], io dtype.
 *   loss:   device float[1], receives (1/n) sum (o - target)^2 over all
 *           n = B*H*T*dv elements (0 when n == 0).
 *   dO:     nullable, [B, H, T, dv], io dtype: receives dloss/do =
 *           2 (o - target) / n, the dO that lz_hybrid_bwd takes.
 * With bf16 I/O and dk = dv = 128 the loss and dO are formed in the output
 * kernel's epilogue from the fp32 output before it is rounded to bf16;
 * otherwise a separate kernel reads the stored output.  The partial sums are
 * added in a fixed order, so the loss is the same bit for bit on every run.
 * dO must not overlap o.  Scratch: lz_workspace_bytes(d, LZ_WS_HYBRID_FWD_MSE).
 * All other arguments as in lz_hybrid_fwd. */
lz_status lz_hybrid_fwd_mse(const lz_dims* d, const void* q, const void* k,
                            const void* v, const float* g, const void* meta_k,
                            const void* meta_v, const float* h0,
                            const void* target, void* o, float* hT, float* lse,
                            void* o_swa, void* chunk_states, float* loss, void* dO,
                            void* ws, size_t ws_bytes, lz_stream stream);

/* Gradient of lz_gla_fwd (needed by the attention-distillation stage,
 * section 2b).  dO = dL/do; dhT (nullable) = dL/dhT.  Writes dq, dk, dv (io
 * dtype), dg (fp32; dL/dz of the gate logits when d->gate_logits) and dh0
 * (nullable, fp32).  h0 may be NULL (zeros).
 * chunk_states (nullable): the forward's chunk states for these inputs;
 * with them the backward skips its own state pass, and then hT (the
 * forward's final state) must be given too when dhT is. */
lz_status lz_gla_bwd(const lz_dims* d, const void* q, const void* k,
                     const void* v, const float* g, const float* h0,
                     const void* dO, const float* dhT, const void* chunk_states,
                     const float* hT, void* dq, void* dk, void* dv, float* dg,
                     float* dh0, void* ws, size_t ws_bytes, lz_stream stream);

/* Gradient of lz_swa_meta_fwd.  dO = dL/d(o_swa); lse from the forward.
 * o (nullable) is the forward's output o_swa: when given, the softmax
 * backward's row term D_t = dO_t . o_t is read off it (the bf16 tensor-core
 * path then walks the window once instead of twice); when NULL it is
 * rebuilt from the scores.  Both give the same result up to rounding.
 * Writes dq, dk, dv (io dtype) and, when M > 0, dmeta_k (fp32, summed over
 * batch and sequence) and dmeta_v (fp32; ignored in sink-only mode). */
lz_status lz_swa_meta_bwd(const lz_dims* d, const void* q, const void* k,
                          const void* v, const void* meta_k,
                          const void* meta_v, const float* lse,
                          const void* o, const void* dO, void* dq, void* dk,
                          void* dv, float* dmeta_k, float* dmeta_v, void* ws,
                          size_t ws_bytes, lz_stream stream);

/* Scratch-free variant of lz_swa_meta_bwd, for callers that cannot allocate
 * device memory when they run the backward (for example an engine plugin
 * whose enqueue step must not call cudaMalloc, or a host framework that has
 * reserved all device memory for its own pool).  The paper has no
 * counterpart: this is a deployment convenience.
 *
 * Arguments, layouts and results are those of lz_swa_meta_bwd; the scratch
 * comes from a static device array of LZ_NOALLOC_SCRATCH_BYTES (16 MiB) that
 * the library holds on every GPU that loads it until the process exits.
 * A problem whose lz_workspace_bytes(d, LZ_WS_SWA_BWD) exceeds that size is
 * rejected with LZ_ERR_UNSUPPORTED (nothing launched).  The call allocates
 * nothing (no cudaMalloc/cudaFree, no allocating library routine).
 *
 * The first call on a device (the device current on the calling thread,
 * which must be the stream's device) looks up the array's device address
 * once; make that first call before any stream capture.  With lazy module
 * loading (the CUDA 12 default) that first call is also where the library's
 * module, and with it the 16 MiB array, is loaded onto the device: it can
 * fail with LZ_ERR_CUDA if the device's memory is exhausted, so a caller
 * that pools all device memory should make it before reserving its pool.
 * Later calls reserve nothing more.  After cudaDeviceReset the array is gone
 * and this entry point must not be used again in the process.  Invalid
 * dims are rejected before the device is touched.  All calls share
 * the one array: calls that may overlap on the GPU (different streams, or
 * several host threads, on the same device) race and must be serialized by
 * the caller.  The array keeps the previous call's contents; every part of
 * it is written before it is read, so nothing needs clearing. */
#define LZ_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
lz_status lz_swa_meta_bwd_noalloc(const lz_dims* d, const void* q,
                                  const void* k, const void* v,
                                  const void* meta_k, const void* meta_v,
                                  const float* lse, const void* o,
                                  const void* dO, void* dq, void* dk, void* dv,
                                  float* dmeta_k, float* dmeta_v,
                                  lz_stream stream);

/* Gradient of lz_hybrid_fwd in one call: the gated branch sees dO, the
 * window branch alpha * dO.  lse from the forward; o_swa (nullable) the
 * forward's window output, used as in lz_swa_meta_bwd; chunk_states and hT
 * (nullable) the forward's, used as in lz_gla_bwd.  dalpha (nullable, one
 * fp32) receives sum over (b,h,t) of dO_t . o_swa_t.
 * On the bf16, dk = dv = 128 path the part of the gated backward that reads
 * only the inputs (the reverse scan of the state gradient) runs on the side
 * stream, forked from `stream` by an event and joined back by another before
 * the gradients are written, so it overlaps the window backward; to the
 * caller the call is still ordered on `stream` alone (also under CUDA graph
 * capture). */
lz_status lz_hybrid_bwd(const lz_dims* d, const void* q, const void* k,
                        const void* v, const float* g, const void* meta_k,
                        const void* meta_v, const float* h0, const float* lse,
                        const void* o_swa, const void* chunk_states,
                        const float* hT, const void* dO, const float* dhT,
                        void* dq, void* dk,
                        void* dv, float* dg, float* dh0, float* dmeta_k,
                        float* dmeta_v, float* dalpha, void* ws,
                        size_t ws_bytes, lz_stream stream);

/* One constant-memory generation step for Bd sequences (section 2a: the
 * fixed-size state replaces the growing KV cache), all in place:
 *   state [Bd,H,dk,dv] fp32; kring [Bd,H,w,dk], vring [Bd,H,w,dv] (io
 *   dtype); pos [Bd] int64 = tokens seen so far per sequence.
 * Per sequence with p = pos[b]: k, v go to ring slot p mod w; the state is
 * decayed by exp(g) and gets k v^T; o_gla = q^T S; the window is the last
 * min(p+1, w) tokens (the new one included) plus the M meta tokens; o =
 * o_gla + alpha * o_swa; pos[b] = p + 1.  Sequences may sit at different
 * positions.  One kernel launch per call: the H blocks of a sequence read
 * and advance pos[b] with 64-bit atomics, using its bits 48..62 as an arrival
 * count during the call, so pos[b] must lie in [0, 2^48) and 8-byte aligned
 * (a value outside that range gives undefined results, with every memory
 * access still in bounds); calls that overlap on the GPU and share pos race.
 *   q, k [Bd,H,dk], v, o [Bd,H,dv] io dtype; g [Bd,H,dk] fp32.  meta_v NULL
 *   = sink-only.  Supported: dk = dv = 128, H <= 32767, io = LZ_BF16 or
 *   LZ_F32. */
lz_status lz_gla_decode_step(int Bd, int H, int dk, int dv, int w, int M,
                             lz_dtype io, float scale, float alpha,
                             float* state, void* kring, void* vring,
                             int64_t* pos, const void* q, const void* k,
                             const void* v, const float* g,
                             const void* meta_k, const void* meta_v, void* o,
                             lz_stream stream);

/* Hand-off from a prefill to lz_gla_decode_step (section 2a: generation
 * continues from the fixed-size state and the last w keys/values).  For Bd
 * prompts of L_b tokens: state = hT (the prefill's final state from
 * lz_gla_fwd / lz_hybrid_fwd, [Bd,H,dk,dv] fp32; NULL = zeros); ring slot
 * (t mod w) = k_t, v_t for the last min(L_b, w) prompt tokens (k, v
 * [Bd,H,T,dk/dv] io dtype, the prefill's layout); pos[b] = L_b.  Ring slots
 * not written keep their contents (the decode step never reads them).
 *   lens: [Bd] int64 device array of prompt lengths L_b (clamped to
 *   [0, T]), or NULL for L_b = T.  Prompts of different lengths share one
 *   prefill by right-padding to T with k = 0 and g = 0 (log-gate 0, i.e. no
 *   decay): the padded tokens then leave the state unchanged, so hT is each
 *   prompt's state after its own L_b tokens (q and v of the padding are
 *   free; their outputs are to be ignored).
 * Supported: dk = dv = 128, 1 <= w <= 1024. */
lz_status lz_decode_prefill(int Bd, int H, int T, int dk, int dv, int w,
                            lz_dtype io, const void* k, const void* v,
                            const int64_t* lens, const float* hT,
                            float* state, void* kring, void* vring,
                            int64_t* pos, lz_stream stream);

/* The projections in front of the operator (section 2a: the gate is
 * Gamma_i = sigma(W_gamma x_i) and the state update takes phi(k_i); the pages
 * do not define phi, read here as the identity, the featurised keys being
 * the operator's input).  From hidden states x [B,T,Dm] (bf16, row-major)
 * and weights W [H*dk, Dm] (bf16, one row per output feature, as a linear
 * layer stores them), one launch computes any of
 *   q = x Wq^T,  k = x Wk^T  -> [B,H,T,dk] bf16 (rounded once),
 *   g = gate_scale * log sigma(x Wg^T) -> [B,H,T,dk] fp32 log-gates,
 * on tcgen05 tensor cores (fp32 accumulation), the gate's logit never
 * leaving the chip.  A NULL weight skips its output (its output pointer must
 * then be NULL too).  Requirements: Dm a multiple of 8, dk = 64 or 128, H*dk
 * a multiple of 256, gate_scale > 0, 16-byte aligned pointers.  Caller-owned
 * device memory; asynchronous on `stream`; bad arguments return
 * LZ_ERR_INVALID_ARG / LZ_ERR_UNSUPPORTED before any launch.  A bounded
 * device wait that gives up is reported by lz_device_check. */
lz_status lz_qkg_projection(int B, int T, int Dm, int H, int dk, const void* x,
                            const void* Wq, const void* Wk, const void* Wg,
                            float gate_scale, void* q, void* k, float* g,
                            lz_stream stream);

/* ---- Context parallelism: one sequence over R ranks ----------------------
 * The pages run each layer on one device; splitting a long sequence into R
 * contiguous segments (rank r holds tokens [r Ts, (r+1) Ts) of every
 * (batch, head)) rests on section 2a's state update S_t = Gamma_t S_{t-1} +
 * k_t v_t^T being linear: a segment maps the state it receives to
 * diag(E) h + S, with E the product of its gates per key dim and S its
 * final state from a zero start.  These three calls are that arithmetic;
 * moving data between ranks is the caller's (e.g. torch.distributed).  All
 * pointers are device memory owned by the caller; calls are asynchronous on
 * `stream`; bad arguments return LZ_ERR_INVALID_ARG / LZ_ERR_UNSUPPORTED
 * before any launch, launch failures LZ_ERR_CUDA. */

/* E[bh][i] = exp(sum over the T tokens of g[bh][t][i]): the segment's gate
 * product per key dim.  g [BH,T,dk] fp32 log-gates, E [BH,dk] fp32 (T = 0
 * gives 1).  dk = 64 or 128; 16-byte aligned pointers. */
lz_status lz_cp_segment_decay(int BH, int T, int dk, const float* g, float* E,
                              lz_stream stream);

/* The fold over segments, elementwise on [BH,dk,dv] fp32 states:
 *   dir 0 (forward): h = init; for q = 0 .. r-1: h = diag(E_q) h + X_q.
 *     With X_q = segment q's final state from a zero start, out is the
 *     state entering segment r (init = the sequence's h0, NULL = 0).
 *   dir 1 (reverse): h = init; for q = R-1 down to r+1: h = X_q + diag(E_q) h.
 *     With X_q = the gradient of segment q's outputs with respect to the
 *     state it received (its dh0 from a backward with dhT = 0), out is the
 *     state gradient leaving segment r (init = the sequence's dhT, NULL = 0).
 * E [R,BH,dk], X [R,BH,dk,dv] (segment-major, as an all-gather stacks them);
 * out [BH,dk,dv] may not alias X.  dv a multiple of 4; 16-byte aligned. */
lz_status lz_cp_fold(int R, int r, int dir, int BH, int dk, int dv,
                     const float* E, const float* X, const float* init,
                     float* out, lz_stream stream);

/* Row-block copy and sum over [BH, rows, d] tensors of the io dtype:
 *   dst[bh][dst_off + t] = a_scale * A[bh][a_off + t] + B[bh][b_off + t]
 * for t < n, with A or B NULL standing for zeros; each tensor has its own
 * row count (a_T, b_T, dst_T).  Summed in fp32, rounded once.  Used to cut
 * the window halo (the last w - 1 rows) out of a segment, to prepend it, and
 * to add the window branch's rows to the gated branch's.  dst may alias A or
 * B row for row (same offsets); other overlaps are not allowed. */
lz_status lz_cp_rows(int BH, int d, lz_dtype io, int n, const void* A,
                     int a_T, int a_off, float a_scale, const void* B,
                     int b_T, int b_off, void* dst, int dst_T, int dst_off,
                     lz_stream stream);

/* Device-side status (no counterpart on the pages; a robustness aid).  The
 * tcgen05 kernels wait on mbarriers for their tensor-core work; every such
 * wait is bounded (0.2 s) and, when it gives up, adds one to a status word
 * of the library on that device instead of spinning on (the kernel then
 * skips the rest of its work and releases its tensor memory).
 * lz_device_check synchronizes `stream`, reads and clears the word of the
 * current device and returns LZ_ERR_TIMEOUT if any wait gave up since the
 * last check (LZ_OK otherwise; LZ_ERR_CUDA if the read failed). */
lz_status lz_device_check(lz_stream stream);

/* Test hook of that failure path: launches one block on `stream` that waits
 * on an mbarrier nothing arrives on.  The wait gives up after its 0.2 s limit
 * and counts itself in the status word, so the next lz_device_check returns
 * LZ_ERR_TIMEOUT (and clears it); the device stays usable.  Asynchronous;
 * LZ_ERR_CUDA if the launch failed. */
lz_status lz_selftest_bounded_wait(lz_stream stream);

/* Kernel choice for the calling host thread (no counterpart on the pages).
 * bf16 with dk = dv = 128 has tcgen05 kernels with TMA-fed operands and
 * accumulators in tensor memory (the default) and warp-level mma.sync
 * kernels: the window forward uses tcgen05 for w <= 129 (the scores of the
 * whole band fit in tensor memory) and the key side of the window backward
 * (dk, dv) for every w.  lz_prefer_tcgen05(0) selects the warp-level
 * kernels; both give the same result up to rounding.  Returns the previous
 * setting; never fails. */
int lz_prefer_tcgen05(int on);

/* tcgen05 kernels where the warp-level ones measured faster on B200, for the
 * calling host thread (no counterpart on the pages; default off).  With
 * lz_tcgen05_all(1):
 *  - the gated backward's per-chunk gradients run on a tcgen05 kernel over
 *    128-token chunks (TMA-fed operands, every contraction with M = 128 and
 *    its accumulator in tensor memory) for every chunk whose fp32 log-gates
 *    decay each 64-token half by at most e^-60 in every key dim
 *    (faster-decaying chunks, and gates given as logits under
 *    lz_fused_gate_logits(1), stay on the
 *    warp-level kernel over 64-token chunks);
 *  - the query side of the window backward (dq, D, the meta-gradient and
 *    dalpha partials) runs on a tcgen05 kernel when lz_prefer_tcgen05 is on,
 *    w <= 129, M <= 16 and the forward's window output is given.
 * Both choices give the same result up to rounding.  Returns the previous
 * setting; never fails. */
int lz_tcgen05_all(int on);

/* How gates given as logits (lz_dims.gate_logits = 1) reach the gated
 * kernels, for the calling host thread (no counterpart on the pages; default
 * off).  Off: one pass maps the logits to fp32 log-gates in the call's
 * workspace (the gated and hybrid workspaces hold B*H*T*dk floats for them
 * whenever gate_logits is set) and the backward maps dL/dg to dL/dz in one
 * more pass over dg.  On: every gated kernel maps the logits itself as it
 * reads them (fewer bytes, more special-function work; measured slower on
 * B200).  Both give the same result up to rounding.  Returns the previous
 * setting; never fails. */
int lz_fused_gate_logits(int on);

/* Per-launch device timing for benchmarks (no counterpart on the pages; a
 * measurement aid).  lz_timing_enable(1) makes every later kernel launch of
 * this library from the calling host thread record a pair of CUDA events
 * around itself on its own stream; lz_timing_enable(0) stops it (the
 * default).  lz_timing_read waits for the recorded launches, writes up to
 * max_records kernel names (NUL-terminated, name_stride bytes apart; names
 * may be NULL) and elapsed milliseconds (ms may be NULL), clears the record
 * and returns how many launches were recorded.  lz_timing_only(name)
 * narrows the timing to the launches of that kernel name (as lz_timing_read
 * reports it; NULL or "" times every launch again), so that a benchmark can
 * time one kernel inside a step without an event pair around every other
 * launch.  All three return 0 / a count and never fail; the settings are per
 * host thread. */
int lz_timing_enable(int on);
int lz_timing_only(const char* name);
int lz_timing_read(char* names, size_t name_stride, float* ms, int max_records);

/* Thread-local description of the last non-OK status ("" if none). */
const char* lz_last_error(void);

/* Library version string. */
const char* lz_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LIZARD_H */
