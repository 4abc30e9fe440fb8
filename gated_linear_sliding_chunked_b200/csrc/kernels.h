// Internal launch interface between the C ABI (lizard_api.cu) and the
// kernels.  Not part of the public header.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace lz {

// Brackets one kernel launch with CUDA events when lz_timing_enable(1) is in
// effect on the calling thread (see timing.cu); a no-op otherwise.
class ScopedTiming {
 public:
  ScopedTiming(const char* name, cudaStream_t s);
  ~ScopedTiming();
  ScopedTiming(const ScopedTiming&) = delete;
  ScopedTiming& operator=(const ScopedTiming&) = delete;

 private:
  cudaStream_t s_;
  bool on_;
  const char* name_ = nullptr;
  cudaEvent_t a_ = nullptr, b_ = nullptr;
};

// Records `message` as the thread's last error and returns `status`.
int set_last_error(int status, const char* message);

// Device address of the library's status word on the current device: the
// tcgen05 kernels add one per bounded wait that gave up.  NULL if the
// address cannot be had (the caller then refuses to launch).
unsigned int* device_status_word();

// ---- gated branch, SIMT path (fp32 arithmetic; fp32 or bf16 I/O) ----------
struct GlaFwdParams {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* h0;     // nullable
  void* o;             // nullable: skip outputs (state pass only)
  float* hT;           // nullable
  float* states;       // nullable: [BH][nchunks][dk][dv] state before each chunk
  void* states16;      // nullable (tensor-core kernel): the same in bf16, 64-token chunks
  const float* add;    // nullable: fp32 [B,H,T,dv], o += alpha * add
  const void* add16;   // nullable (tensor-core kernel): the same in bf16; may alias o
  float alpha;
  int B, H, T, dk, dv;
  void* delta16;       // nullable scratch of the two-level state pass: [BH][nchunks][dk][dv] bf16
  float* decay;        // and [BH][nchunks][dk] fp32
  // stage-1 distillation loss, fused into the output pass's epilogue (bf16
  // path): target [B,H,T,dv] (nullable = no loss); loss_part[bh * nchunks + c]
  // receives each chunk's sum of (o - target)^2 taken on the fp32 output;
  // dO_loss (nullable) receives loss_scale * (o - target)
  const void* target;
  void* dO_loss;
  float loss_scale;
  float* loss_part;
  // gate logits (tensor-core kernels): when set, g is NULL and the log-gate
  // is gs * log sigma(gz) with gz bf16 [B,H,T,dk]
  const void* gz;
  float gs;
  int wave;  // CTAs resident at once (0: no prefetch of the next wave's inputs)
};
constexpr int kSimtChunk = 16;
cudaError_t launch_gla_fwd_simt(const GlaFwdParams& p, bool bf16, cudaStream_t s);

// ---- gated branch, tensor-core forward (bf16 I/O, dk = 128) --------------
// Same params; `states` (if set) receives the fp32 state before every
// 64-token chunk: [BH][ceil(T/64)][dk][dv].
bool gla_fwd_mma_supported(int dk, int dv, bool bf16);
int gla_fwd_mma_chunk();
cudaError_t launch_gla_fwd_mma(const GlaFwdParams& p, cudaStream_t s);

struct GlaBwdParams {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const void* dO;
  const float* dhT;      // nullable
  const float* states;   // [BH][nchunks][dk][dv] from the state pass
  const void* states16;  // tensor-core kernel: bf16 states per 64-token chunk
  const float* hT;       // [BH][dk][dv] final state (read only when dhT != NULL)
  const float* add_dq;   // nullable fp32 [B,H,T,dk] added before the store
  const float* add_dk;   // nullable
  const float* add_dv;   // nullable fp32 [B,H,T,dv]
  bool add_in_place;     // tensor-core kernel: dq, dk, dv already hold bf16 terms to add
  void* dq;
  void* dk;
  void* dv;
  float* dg;
  float* dh0;            // nullable
  int B, H, T, dkd, dvd;
  const void* gin16;     // two-level tensor-core backward: launch_gla_bwd_scan's outputs
  const float* gsp;
  const void* gz;        // gate logits (see GlaFwdParams); dg then receives dL/dz
  float gs;
  const int* tc_flags;   // nullable: [BH][ceil(T/128)] from launch_gla_bwd_tc; the
                         // per-64-row kernel then runs only the chunks flagged 1
  unsigned int* status;  // device status word (tcgen05 kernel; set by its launcher)
};
cudaError_t launch_gla_bwd_simt(const GlaBwdParams& p, bool bf16, cudaStream_t s);

// ---- gated branch, two-pass tensor-core forward (bf16, dk = dv = 128) -----
// launch_gla_states writes states16 ([BH][ceil(T/64)][dk][dv] bf16, the state
// before every 64-token chunk) and hT; launch_gla_out then computes o (adding
// alpha * add16 when set) from them, all chunks in parallel.
bool gla_chunk_mma_supported(int dk, int dv, bool bf16);
cudaError_t launch_gla_states(const GlaFwdParams& p, cudaStream_t s);
// whether launch_gla_states takes the two-level path (given delta16 / decay)
bool gla_states_scan_wanted(int T);
cudaError_t launch_gla_out(const GlaFwdParams& p, cudaStream_t s);
// gates given as bf16 logits z: g = gs * log sigma(z) into fp32 (n elements,
// a multiple of 8), and dL/dg -> dL/dz = dL/dg * gs * sigma(-z) in place
cudaError_t launch_gate_logits_to_log(const void* z, float* g, size_t n, float gs, cudaStream_t s);
cudaError_t launch_gate_dlogit(float* dg, const void* z, size_t n, float gs, cudaStream_t s);

// ---- gated backward, two-level (bf16, dk = dv = 128) ------------------------
// launch_gla_bwd_scan: every chunk's dG_c = (q e^{b})^T dO and decay e^{b_l}
// in parallel, then a reverse elementwise scan writing gin16[c] (the state
// gradient entering chunk c from the later chunks, bf16), gsp[c][i] =
// <G_new, S_prev>_i (the gate gradient at the chunk's first row) and dh0.
// launch_gla_bwd_chunks then computes every chunk's dq, dk, dv, dg from
// them, all chunks in parallel.
struct GlaBwdScanParams {
  const void* q;
  const void* dO;
  const float* g;
  const void* states16;  // the forward's states before every 64-token chunk
  const float* dhT;      // nullable
  void* delta16;         // scratch [BH][nchunks][dk][dv] bf16
  float* decay;          // scratch [BH][nchunks][dk]
  void* gin16;           // [BH][nchunks][dk][dv] bf16
  float* gsp;            // [BH][nchunks][dk]
  float* dh0;            // nullable
  int B, H, T;
  const void* gz;        // gate logits (see GlaFwdParams)
  float gs;
};
cudaError_t launch_gla_bwd_scan(const GlaBwdScanParams& p, cudaStream_t s);
// partial sums the fused loss epilogue writes: one per 64-token chunk and head
size_t gla_out_loss_parts(int B, int H, int T);

// ---- stage-1 distillation loss (loss.cu) ------------------------------------
// Any layout: n elements of o and target (bf16 or fp32); part[0, nparts)
// receives block partial sums of (o - target)^2 in a fixed order; dO
// (nullable) receives scale * (o - target).
constexpr int kMseParts = 592;  // 4 blocks per SM on 148 SMs
cudaError_t launch_mse_generic(const void* o, const void* target, void* dO, float scale, size_t n,
                               bool bf16, float* part, cudaStream_t s);
int mse_generic_parts(size_t n);
// loss[0] = inv_n * (sum of part[0, nparts)), summed in fp64 in a fixed order
cudaError_t launch_loss_reduce(const float* part, size_t nparts, double inv_n, float* loss,
                               cudaStream_t s);

// ---- gated branch, tensor-core backward (bf16 I/O, dk = dv = 128) --------
// Needs states16 (the forward's states before every 64-token chunk) and
// launch_gla_bwd_scan's gin16 / gsp; all chunks in parallel.
bool gla_bwd_mma_supported(int dk, int dv, bool bf16);
cudaError_t launch_gla_bwd_chunks(const GlaBwdParams& p, cudaStream_t s);
// The same gradients on tcgen05 for 128-token chunks whose gates keep each
// 64-row half's decay within e^-60 in every key dim (fp32 log-gates, bf16,
// dk = dv = 128, after launch_gla_bwd_scan): flags[bh][c] = 0 for a chunk it
// computed, 1 for one it left to launch_gla_bwd_chunks (run next with
// p.tc_flags = flags).
bool gla_bwd_tc_supported(const GlaBwdParams& p);
int gla_bwd_tc_nchunks(int T);
cudaError_t launch_gla_bwd_tc(const GlaBwdParams& p, int* flags, cudaStream_t s);

// ---- window + meta softmax, SIMT path ------------------------------------
struct SwaFwdParams {
  const void* q;
  const void* k;
  const void* v;
  const void* mk;   // [H,M,dk] (nullable when M == 0)
  const void* mv;   // nullable = sink-only
  void* o;          // nullable, io dtype
  float* o_f32;     // nullable, fp32
  float* lse;       // nullable
  int B, H, T, dk, dv, w, M;
  float scale;
  unsigned int* status;  // device status word (set by the tcgen05 launcher)
};
cudaError_t launch_swa_fwd_simt(const SwaFwdParams& p, bool bf16, cudaStream_t s);
// warp-level tensor-core forward (bf16 I/O, dk = dv = 128)
bool swa_fwd_mma_supported(int dk, int dv, bool bf16);
cudaError_t launch_swa_fwd_mma(const SwaFwdParams& p, cudaStream_t s);
// tcgen05 forward (bf16 I/O, dk = dv = 128, w <= 129)
bool swa_fwd_tc_supported(int dk, int dv, bool bf16, int w);
cudaError_t launch_swa_fwd_tc(const SwaFwdParams& p, cudaStream_t s);

struct SwaBwdParams {
  // the hybrid backward's overlap: an event (cudaEvent_t) recorded right after
  // the query-side launch, and the partials' reduction left to the caller
  // (launch_swa_bwd_mma_reduce) on another stream
  void* query_done = nullptr;
  bool defer_reduce = false;
  const void* q;
  const void* k;
  const void* v;
  const void* mk;
  const void* mv;
  const float* lse;
  const void* osw;   // nullable: the window branch's forward output; when given
                     // D_t = dO_t . osw_t is read off it instead of recomputed
  const void* dO;
  float gscale;      // the window branch sees gscale * dO
  void* dq;          // io dtype outputs (nullable when the f32 ones are used)
  void* dk;
  void* dv;
  float* dq_f32;     // nullable fp32 outputs
  float* dk_f32;
  float* dv_f32;
  float* Dbuf;       // [B*H*T] scratch: dO_t . o_swa_t (unscaled)
  float* alpha_part; // [n_qblocks] scratch: per-block sums of Dbuf
  float* meta_part;  // [n_meta_parts][H][M][dk+dv] scratch
  float* dmk;        // nullable [H,M,dk]
  float* dmv;        // nullable [H,M,dv]
  float* dalpha;     // nullable [1]
  int B, H, T, dkd, dvd, w, M;
  float scale;
  bool tc;               // key side on the tcgen05 kernel (bf16, d = 128)
  bool tc_q;             // query side on the tcgen05 kernel where it applies
  unsigned int* status;  // device status word (set by the tcgen05 launcher)
  // Split query side (used when both are set, the key side runs on tcgen05,
  // the forward output is given and dq is bf16): the key side also stores its
  // bf16 dS^T tiles, the query-side pass keeps only D, the meta tokens' dS and
  // the meta gradients, and swa_bwd_dq forms dq = scale * gscale * dS [K; MK].
  void* ds_tiles;        // [B*H][ceil(T/128)][ds_nq][128 keys][64 queries] bf16
  void* ds_meta;         // [B*H][T][16] bf16: the meta tokens' dS / gscale
  int ds_nq;             // query tiles per 128-key block (swa_bwd_ds_nq(w))
};
// query rows per CTA of the meta-gradient pass (one partial per slab)
constexpr int kSwaBwdSlab = 256;
// 64-query tiles that see one 128-key block of a window of w keys
inline int swa_bwd_ds_nq(int w) { return (127 + w - 1 + 64) / 64; }
int swa_bwd_n_qblocks(int B, int H, int T);
int swa_bwd_n_meta_parts(int B, int T);
cudaError_t launch_swa_bwd_simt(const SwaBwdParams& p, bool bf16, cudaStream_t s);
// fixed-order sums of the meta-gradient and dalpha partials
cudaError_t launch_swa_bwd_reduce(const SwaBwdParams& p, int nparts, int nalpha, cudaStream_t s);
// tensor-core backward (bf16 I/O, dk = dv = 128); same scratch layout
bool swa_bwd_mma_supported(int dk, int dv, bool bf16);
cudaError_t launch_swa_bwd_mma(const SwaBwdParams& p, cudaStream_t s);
// the partials' reduction of launch_swa_bwd_mma (when it was deferred)
cudaError_t launch_swa_bwd_mma_reduce(const SwaBwdParams& p, cudaStream_t s);
// key side (dk, dv) on tcgen05 with TMA-fed operands
bool swa_bwd_kv_tc_supported(int dk, int dv, bool bf16);
cudaError_t launch_swa_bwd_kv_tc(const SwaBwdParams& p, cudaStream_t s);
// query side (dq, D, meta-gradient and dalpha partials) on tcgen05: bf16,
// dk = dv = 128, w <= 129, M <= 16, the forward output (osw) given
bool swa_bwd_q_tc_supported(const SwaBwdParams& p);
cudaError_t launch_swa_bwd_q_tc(const SwaBwdParams& p, cudaStream_t s);

// ---- decode --------------------------------------------------------------
struct DecodeParams {
  int Bd, H, w, M;
  float scale, alpha;
  float* state;
  void* kring;
  void* vring;
  int64_t* pos;
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const void* mk;
  const void* mv;
  void* o;
};
struct DecodePrefillParams {
  int Bd, H, T, w;
  const void* k;     // [Bd,H,T,128] io dtype
  const void* v;
  const float* hT;   // [Bd,H,128,128], nullable = zeros
  float* state;
  void* kring;
  void* vring;
  int64_t* pos;
  const int64_t* lens;  // [Bd] prompt lengths, nullable = all T
};
cudaError_t launch_decode_prefill(const DecodePrefillParams& p, bool bf16, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams& p, bool bf16, cudaStream_t s);

}  // namespace lz
