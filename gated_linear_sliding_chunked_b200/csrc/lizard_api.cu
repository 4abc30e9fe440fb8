// C ABI of the hybrid attention library: argument validation, workspace
// layout and kernel launches.  Every entry point validates on the host and
// returns before any launch when an argument is bad; kernels never trap.
#include <cstdarg>
#include <cstdio>
#include <string>
#include <unordered_map>

#include "../../include/lizard.h"
#include "kernels.h"

namespace {

thread_local std::string g_err;
thread_local bool g_prefer_tc = true;  // lz_prefer_tcgen05
thread_local bool g_tc_all = false;  // lz_tcgen05_all
thread_local bool g_fused_logits = false;  // lz_fused_gate_logits

// The window branch's forward for bf16 with dk = dv = 128: tcgen05 for
// w <= 129 (unless the calling thread asked for the warp-level kernel),
// warp-level MMA otherwise; fp32 SIMT for the other shapes.
cudaError_t swa_forward(const lz::SwaFwdParams& p, bool bf16, cudaStream_t s) {
  if (g_prefer_tc && lz::swa_fwd_tc_supported(p.dk, p.dv, bf16, p.w)) return lz::launch_swa_fwd_tc(p, s);
  if (lz::swa_fwd_mma_supported(p.dk, p.dv, bf16)) return lz::launch_swa_fwd_mma(p, s);
  return lz::launch_swa_fwd_simt(p, bf16, s);
}

// The window branch's backward: tensor cores for bf16 with dk = dv = 128.
cudaError_t swa_backward(const lz::SwaBwdParams& p, bool bf16, cudaStream_t s) {
  if (lz::swa_bwd_mma_supported(p.dkd, p.dvd, bf16)) return lz::launch_swa_bwd_mma(p, s);
  return lz::launch_swa_bwd_simt(p, bf16, s);
}

// The forward of the gated branch.  bf16 with dk = dv = 128: a state pass
// (bf16 states into `states16` scratch) then all chunks' outputs in
// parallel; bf16 with dk = 128 and other dv: the single-pass tensor-core
// kernel; otherwise fp32 SIMT.
// Scratch of the two-level state pass (long sequences): per-chunk increments
// and decays; both NULL when the sequential pass is used.
struct ScanWs {
  void* delta16 = nullptr;
  float* decay = nullptr;
};

cudaError_t gla_forward(lz::GlaFwdParams p, bool bf16, void* states16, ScanWs scan, cudaStream_t s) {
  if (lz::gla_chunk_mma_supported(p.dk, p.dv, bf16)) {
    p.states16 = states16;
    p.delta16 = scan.delta16;
    p.decay = scan.decay;
    cudaError_t e = lz::launch_gla_states(p, s);
    if (e != cudaSuccess) return e;
    return lz::launch_gla_out(p, s);
  }
  if (p.o && lz::gla_fwd_mma_supported(p.dk, p.dv, bf16)) return lz::launch_gla_fwd_mma(p, s);
  return lz::launch_gla_fwd_simt(p, bf16, s);
}

// A high-priority stream and two events per (host thread, device), created on
// first use and kept for the life of the process.  lz_hybrid_fwd forks the
// gated state pass onto it while the window forward runs; lz_hybrid_bwd forks
// the gated backward's first phase onto it while the window backward runs.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr;
  cudaEvent_t join = nullptr;
  cudaEvent_t mid = nullptr;  // lz_hybrid_bwd: the window backward's query side done
};

static cudaError_t side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  thread_local std::unordered_map<int, SideStream> streams;
  SideStream& ss = streams[dev];
  if (!ss.stream) {
    int lo = 0, hi = 0;
    e = cudaDeviceGetStreamPriorityRange(&lo, &hi);
    if (e != cudaSuccess) return e;
    e = cudaStreamCreateWithPriority(&ss.stream, cudaStreamNonBlocking, hi);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ss.mid, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      ss = SideStream{};
      return e;
    }
  }
  *out = &ss;
  return cudaSuccess;
}

lz_status fail(lz_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

lz_status ok() {
  g_err.clear();
  return LZ_OK;
}

}  // namespace

namespace lz {
// Lets other translation units of the library report a failure through
// lz_last_error().
int set_last_error(int status, const char* message) {
  g_err = message ? message : "";
  return status;
}
}  // namespace lz

namespace {

lz_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(LZ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Carves consecutive 256-byte aligned regions out of the caller's scratch.
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += round_up(count * sizeof(T));
    return p;
  }
};

#define LZ_REQUIRE(cond, ...)                                  \
  do {                                                         \
    if (!(cond)) return fail(LZ_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

lz_status check_ptr(const void* p, const char* name, bool required) {
  if (!p) {
    if (required) return fail(LZ_ERR_INVALID_ARG, "%s must not be NULL", name);
    return LZ_OK;
  }
  if (!aligned16(p)) return fail(LZ_ERR_INVALID_ARG, "%s must be 16-byte aligned", name);
  return LZ_OK;
}

#define LZ_PTR(p, req)                                   \
  do {                                                   \
    lz_status _s = check_ptr((p), #p, (req));            \
    if (_s != LZ_OK) return _s;                          \
  } while (0)

// Shape checks shared by the prefill/training entry points.
lz_status check_dims(const lz_dims* d, bool need_window) {
  LZ_REQUIRE(d != nullptr, "dims must not be NULL");
  LZ_REQUIRE(d->B >= 0 && d->H >= 0 && d->T >= 0, "B, H, T must be >= 0 (got %d, %d, %d)",
             d->B, d->H, d->T);
  if (d->io != LZ_F32 && d->io != LZ_BF16)
    return fail(LZ_ERR_UNSUPPORTED, "io dtype %d is not LZ_F32 or LZ_BF16", (int)d->io);
  if ((d->dk != 64 && d->dk != 128) || (d->dv != 64 && d->dv != 128))
    return fail(LZ_ERR_UNSUPPORTED, "dk, dv must be 64 or 128 (got %d, %d)", d->dk, d->dv);
  if (d->chunk != 64 && d->chunk != 128)
    return fail(LZ_ERR_UNSUPPORTED, "chunk must be 64 or 128 (got %d)", d->chunk);
  if (need_window) {
    if (d->w < 1 || d->w > 1024)
      return fail(LZ_ERR_UNSUPPORTED, "window w must be in [1, 1024] (got %d)", d->w);
    if (d->M < 0 || d->M > 16)
      return fail(LZ_ERR_UNSUPPORTED, "meta tokens M must be in [0, 16] (got %d)", d->M);
  }
  LZ_REQUIRE(d->gate_logits == 0 || d->gate_logits == 1, "gate_logits must be 0 or 1 (got %d)",
             d->gate_logits);
  if (d->gate_logits) {
    if (d->io != LZ_BF16 || d->dk != 128 || d->dv != 128)
      return fail(LZ_ERR_UNSUPPORTED, "gate logits need bf16 I/O and dk = dv = 128");
    LZ_REQUIRE(d->gate_scale > 0.f && d->gate_scale < 3.0e38f, "gate_scale must be finite and > 0");
  }
  const double elems = (double)d->B * d->H * d->T * (d->dk > d->dv ? d->dk : d->dv);
  LZ_REQUIRE(elems < 9.0e15, "problem too large");
  return LZ_OK;
}

size_t bht(const lz_dims* d) { return (size_t)d->B * d->H * d->T; }

bool fwd_uses_chunks(const lz_dims* d) {
  return lz::gla_chunk_mma_supported(d->dk, d->dv, d->io == LZ_BF16);
}
// bf16 state before every 64-token chunk (two-pass forward, tensor-core backward)
size_t states16_count(const lz_dims* d) {
  const size_t n64 = (size_t)((d->T + lz::gla_fwd_mma_chunk() - 1) / lz::gla_fwd_mma_chunk());
  return (size_t)d->B * d->H * n64 * d->dk * d->dv;
}
// the two-level state pass's scratch, carved right after the states
// (always carved for the two-level backward, whose first step uses it too)
ScanWs carve_scan(Carver& c, const lz_dims* d, bool always = false) {
  ScanWs w;
  // (gate logits: always, the one-chunk state pass takes only log-gates)
  if (!always && !d->gate_logits && !lz::gla_states_scan_wanted(d->T)) return w;
  const size_t n64 = (size_t)((d->T + lz::gla_fwd_mma_chunk() - 1) / lz::gla_fwd_mma_chunk());
  w.delta16 = c.take<uint16_t>(states16_count(d));
  w.decay = c.take<float>((size_t)d->B * d->H * n64 * d->dk);
  return w;
}
size_t nchunks16(const lz_dims* d) {
  return (size_t)((d->T + lz::kSimtChunk - 1) / lz::kSimtChunk);
}

// ---- workspace layouts ----------------------------------------------------
bool bwd_uses_mma(const lz_dims* d) {
  return lz::gla_bwd_mma_supported(d->dk, d->dv, d->io == LZ_BF16);
}

// Tensor-core hybrid path: the window branch's bf16 results go straight into
// the caller's output buffers and the gated kernels add to them in place.
bool hybrid_uses_mma(const lz_dims* d) {
  const bool bf = d->io == LZ_BF16;
  return lz::gla_fwd_mma_supported(d->dk, d->dv, bf) && lz::swa_fwd_mma_supported(d->dk, d->dv, bf) &&
         lz::swa_bwd_mma_supported(d->dk, d->dv, bf) && lz::gla_bwd_mma_supported(d->dk, d->dv, bf);
}

// Stage-1 loss: fused into the gated output kernel's epilogue on the
// tensor-core path; partial sums per (chunk, head) there, per block of the
// generic loss kernel otherwise.
bool loss_fused(const lz_dims* d) { return hybrid_uses_mma(d) && fwd_uses_chunks(d); }
size_t loss_parts(const lz_dims* d) {
  if (loss_fused(d)) return lz::gla_out_loss_parts(d->B, d->H, d->T);
  return (size_t)lz::mse_generic_parts(bht(d) * d->dv);
}

// Gated backward scratch: the states before every chunk (fp32 per 16-token
// chunk for the SIMT kernel, bf16 per 64-token chunk for the tensor-core
// kernel) and the final state.
struct GlaBwdWs {
  float* states;
  void* states16;
  float* hT;
  ScanWs scan;
  void* gin16;  // two-level backward: state gradient entering every chunk (bf16)
  float* gsp;   // and <G_new, S_prev> per chunk and key dim
  int* tcflags; // per 128-token chunk: left by the tcgen05 kernel to the per-64-row one
};
GlaBwdWs carve_gla_bwd(Carver& c, const lz_dims* d) {
  GlaBwdWs w{};
  const size_t bh = (size_t)d->B * d->H;
  if (bwd_uses_mma(d)) {
    w.states16 = c.take<uint16_t>(states16_count(d));  // bf16
    w.scan = carve_scan(c, d, true);
    w.gin16 = c.take<uint16_t>(states16_count(d));
    const size_t n64 = (size_t)((d->T + lz::gla_fwd_mma_chunk() - 1) / lz::gla_fwd_mma_chunk());
    w.gsp = c.take<float>(bh * n64 * d->dk);
    w.tcflags = c.take<int>(bh * (size_t)lz::gla_bwd_tc_nchunks(d->T));
  } else {
    w.states = c.take<float>(bh * nchunks16(d) * d->dk * d->dv);
  }
  w.hT = c.take<float>(bh * d->dk * d->dv);
  return w;
}

struct SwaBwdWs {
  float* Dbuf;
  float* alpha_part;
  float* meta_part;
};
SwaBwdWs carve_swa_bwd(Carver& c, const lz_dims* d) {
  SwaBwdWs w;
  w.Dbuf = c.take<float>(bht(d));
  w.alpha_part = c.take<float>((size_t)lz::swa_bwd_n_qblocks(d->B, d->H, d->T) + 1);
  w.meta_part = c.take<float>((size_t)lz::swa_bwd_n_meta_parts(d->B, d->T) * d->H * d->M *
                              (d->dk + d->dv) + 1);
  return w;
}

struct HybridBwdWs {
  SwaBwdWs swa;
  GlaBwdWs gla;
  float* dq;  // fp32 window-branch gradients (SIMT path only)
  float* dk;
  float* dv;
  void* ds_tiles;  // tensor-core path: the key side's bf16 dS^T tiles ...
  void* ds_meta;   // ... and the meta tokens' dS, for the split query side
};
HybridBwdWs carve_hybrid_bwd(Carver& c, const lz_dims* d) {
  HybridBwdWs w{};
  w.swa = carve_swa_bwd(c, d);
  w.gla = carve_gla_bwd(c, d);
  if (hybrid_uses_mma(d) && d->w <= 129) {  // windows of up to 129 keys: at most 4 tiles per block
    const size_t nblk = (size_t)((d->T + 127) / 128);
    w.ds_tiles = c.take<uint16_t>((size_t)d->B * d->H * nblk * lz::swa_bwd_ds_nq(d->w) * 128 * 64);
    w.ds_meta = c.take<uint16_t>(bht(d) * 16);
  }
  if (!hybrid_uses_mma(d)) {
    w.dq = c.take<float>(bht(d) * d->dk);
    w.dk = c.take<float>(bht(d) * d->dk);
    w.dv = c.take<float>(bht(d) * d->dv);
  }
  return w;
}

// Gates given as logits: their fp32 log-gates, carved last in the gated and
// hybrid workspaces (the size depends on the dims alone).
float* carve_gates(Carver& c, const lz_dims* d) {
  return d->gate_logits ? c.take<float>(bht(d) * d->dk) : nullptr;
}

// The gates the kernels read.  Logits are mapped once to fp32 log-gates in
// the workspace (g32) and the call proceeds as with log-gates, unless the
// calling thread asked for the kernels that map them on the fly
// (lz_fused_gate_logits); z is then set for the backward to map dL/dg back
// to dL/dz.
struct GateIn {
  lz_dims d;        // the dims the kernels see
  const float* g;   // the gates they read
  const void* z;    // the logits, when they were mapped here
};
cudaError_t gate_input(const lz_dims* d, const float* g, float* g32, cudaStream_t s, GateIn& out) {
  out.d = *d;
  out.g = g;
  out.z = nullptr;
  if (!d->gate_logits || g_fused_logits || g32 == nullptr) return cudaSuccess;
  out.d.gate_logits = 0;
  out.g = g32;
  out.z = g;
  return lz::launch_gate_logits_to_log(g, g32, bht(d) * d->dk, d->gate_scale, s);
}

size_t ws_bytes(const lz_dims* d, int which) {
  Carver c(nullptr);
  switch (which) {
    case LZ_WS_GLA_FWD:
      if (fwd_uses_chunks(d)) {
        c.take<uint16_t>(states16_count(d));
        carve_scan(c, d);
      }
      carve_gates(c, d);
      return c.off;
    case LZ_WS_HYBRID_FWD:
      if (!hybrid_uses_mma(d)) c.take<float>(bht(d) * d->dv);  // fp32 window output
      if (fwd_uses_chunks(d)) {
        c.take<uint16_t>(states16_count(d));
        carve_scan(c, d);
      }
      carve_gates(c, d);
      return c.off;
    case LZ_WS_HYBRID_FWD_MSE:
      c.off = ws_bytes(d, LZ_WS_HYBRID_FWD);
      c.take<float>(loss_parts(d));
      return c.off;
    case LZ_WS_GLA_BWD:
      carve_gla_bwd(c, d);
      carve_gates(c, d);
      return c.off;
    case LZ_WS_SWA_BWD:
      carve_swa_bwd(c, d);
      return c.off;
    case LZ_WS_HYBRID_BWD:
      carve_hybrid_bwd(c, d);
      carve_gates(c, d);
      return c.off;
    case LZ_WS_CHUNK_STATES:
      return fwd_uses_chunks(d) && bwd_uses_mma(d) ? states16_count(d) * sizeof(uint16_t) : 0;
    default:
      return 0;
  }
}

// The forward's chunk states handed to a backward call: used only where the
// kernels keep bf16 chunk states (*states is cleared otherwise); the final
// state must come with them when dL/dhT is given.
lz_status check_saved_states(const lz_dims* d, const float* dhT, const void** states,
                             const float* hT) {
  const void* chunk_states = *states;
  if (chunk_states == nullptr) return LZ_OK;
  LZ_PTR(chunk_states, false);
  if (ws_bytes(d, LZ_WS_CHUNK_STATES) == 0) {
    *states = nullptr;
    return LZ_OK;
  }
  LZ_PTR(hT, dhT != nullptr);
  return LZ_OK;
}

lz_status check_ws(const lz_dims* d, int which, const void* ws, size_t have) {
  const size_t need = ws_bytes(d, which);
  if (need == 0) return LZ_OK;
  LZ_REQUIRE(ws != nullptr, "workspace must not be NULL (%zu bytes needed)", need);
  LZ_REQUIRE(aligned16(ws), "workspace must be 16-byte aligned");
  LZ_REQUIRE(have >= need, "workspace too small: %zu bytes given, %zu needed", have, need);
  return LZ_OK;
}

cudaStream_t as_stream(lz_stream s) { return reinterpret_cast<cudaStream_t>(s); }

lz::SwaFwdParams swa_fwd_params(const lz_dims* d, const void* q, const void* k, const void* v,
                                const void* mk, const void* mv) {
  lz::SwaFwdParams p{};
  p.q = q; p.k = k; p.v = v; p.mk = mk; p.mv = d->M > 0 ? mv : nullptr;
  p.B = d->B; p.H = d->H; p.T = d->T; p.dk = d->dk; p.dv = d->dv; p.w = d->w; p.M = d->M;
  p.scale = d->scale;
  return p;
}

lz::GlaFwdParams gla_fwd_params(const lz_dims* d, const void* q, const void* k, const void* v,
                                const float* g, const float* h0) {
  lz::GlaFwdParams p{};
  p.q = q; p.k = k; p.v = v; p.h0 = h0;
  if (d->gate_logits) {  // `g` carries bf16 logits
    p.gz = g;
    p.gs = d->gate_scale;
  } else {
    p.g = g;
  }
  p.B = d->B; p.H = d->H; p.T = d->T; p.dk = d->dk; p.dv = d->dv;
  return p;
}

lz::SwaBwdParams swa_bwd_params(const lz_dims* d, const void* q, const void* k, const void* v,
                                const void* mk, const void* mv, const float* lse,
                                const void* osw, const void* dO, const SwaBwdWs& w) {
  lz::SwaBwdParams p{};
  p.q = q; p.k = k; p.v = v; p.mk = mk; p.mv = d->M > 0 ? mv : nullptr; p.lse = lse; p.dO = dO;
  p.osw = osw;
  p.tc = g_prefer_tc;
  p.tc_q = g_prefer_tc && g_tc_all;
  p.Dbuf = w.Dbuf; p.alpha_part = w.alpha_part; p.meta_part = w.meta_part;
  p.B = d->B; p.H = d->H; p.T = d->T; p.dkd = d->dk; p.dvd = d->dv; p.w = d->w; p.M = d->M;
  p.scale = d->scale;
  return p;
}

}  // namespace

namespace lz {
// Shape and dtype checks of the window entry points (records the error).
int check_window_dims(const lz_dims* d) { return check_dims(d, true); }
}  // namespace lz

extern "C" {

const char* lz_last_error(void) { return g_err.c_str(); }

const char* lz_version(void) { return "lizard-b200 0.1 (sm_100a)"; }

int lz_prefer_tcgen05(int on) {
  const int prev = g_prefer_tc ? 1 : 0;
  g_prefer_tc = on != 0;
  return prev;
}

int lz_tcgen05_all(int on) {
  const int prev = g_tc_all ? 1 : 0;
  g_tc_all = on != 0;
  return prev;
}

int lz_fused_gate_logits(int on) {
  const int prev = g_fused_logits ? 1 : 0;
  g_fused_logits = on != 0;
  return prev;
}

size_t lz_workspace_bytes(const lz_dims* d, int which) {
  if (check_dims(d, which != LZ_WS_GLA_FWD && which != LZ_WS_GLA_BWD) != LZ_OK) return 0;
  return ws_bytes(d, which);
}

lz_status lz_gla_fwd(const lz_dims* d, const void* q, const void* k, const void* v,
                     const float* g, const float* h0, void* o, float* hT,
                     void* chunk_states, void* ws, size_t ws_bytes_, lz_stream stream) {
  lz_status st = check_dims(d, false);
  if (st != LZ_OK) return st;
  const bool nz = bht(d) > 0;  // empty tensors may have NULL data
  LZ_PTR(q, nz); LZ_PTR(k, nz); LZ_PTR(v, nz); LZ_PTR(g, nz); LZ_PTR(o, nz);
  LZ_PTR(h0, false); LZ_PTR(hT, false); LZ_PTR(chunk_states, false);
  st = check_ws(d, LZ_WS_GLA_FWD, ws, ws_bytes_);
  if (st != LZ_OK) return st;
  const cudaStream_t s = as_stream(stream);
  Carver c(ws);
  void* states16 = fwd_uses_chunks(d) ? c.take<uint16_t>(states16_count(d)) : nullptr;
  const ScanWs scan = fwd_uses_chunks(d) ? carve_scan(c, d) : ScanWs{};
  float* g32 = carve_gates(c, d);
  if (states16 && chunk_states && ws_bytes(d, LZ_WS_CHUNK_STATES) > 0) states16 = chunk_states;
  GateIn gi;
  cudaError_t e = gate_input(d, g, g32, s, gi);
  if (e != cudaSuccess) return cuda_status(e, "lz_gla_fwd (gate logits)");
  lz::GlaFwdParams p = gla_fwd_params(&gi.d, q, k, v, gi.g, h0);
  p.o = o;
  p.hT = hT;
  return cuda_status(gla_forward(p, d->io == LZ_BF16, states16, scan, s), "lz_gla_fwd");
}

lz_status lz_swa_meta_fwd(const lz_dims* d, const void* q, const void* k, const void* v,
                          const void* meta_k, const void* meta_v, void* o, float* lse,
                          lz_stream stream) {
  lz_status st = check_dims(d, true);
  if (st != LZ_OK) return st;
  const bool nz = bht(d) > 0;  // empty tensors may have NULL data
  LZ_PTR(q, nz); LZ_PTR(k, nz); LZ_PTR(v, nz); LZ_PTR(o, nz);
  LZ_PTR(meta_k, d->M > 0 && d->H > 0); LZ_PTR(meta_v, false); LZ_PTR(lse, false);
  lz::SwaFwdParams p = swa_fwd_params(d, q, k, v, meta_k, meta_v);
  p.o = o;
  p.lse = lse;
  return cuda_status(swa_forward(p, d->io == LZ_BF16, as_stream(stream)), "lz_swa_meta_fwd");
}

// The stage-1 loss of lz_hybrid_fwd_mse (NULL for the plain forward).
struct LossArgs {
  const void* target;
  float* loss;
  void* dO;
};

static lz_status hybrid_fwd_impl(const char* name, const lz_dims* d, const void* q, const void* k,
                                 const void* v, const float* g, const void* meta_k,
                                 const void* meta_v, const float* h0, void* o, float* hT,
                                 float* lse, void* o_swa, void* chunk_states, const LossArgs* la,
                                 void* ws, size_t ws_bytes_, lz_stream stream) {
  lz_status st = check_dims(d, true);
  if (st != LZ_OK) return st;
  const bool nz = bht(d) > 0;  // empty tensors may have NULL data
  LZ_PTR(q, nz); LZ_PTR(k, nz); LZ_PTR(v, nz); LZ_PTR(g, nz); LZ_PTR(o, nz);
  LZ_PTR(meta_k, d->M > 0 && d->H > 0); LZ_PTR(meta_v, false); LZ_PTR(h0, false); LZ_PTR(hT, false);
  LZ_PTR(lse, false); LZ_PTR(o_swa, false); LZ_PTR(chunk_states, false);
  if (la) {
    const void* target = la->target;
    const float* loss = la->loss;
    LZ_PTR(target, nz); LZ_PTR(loss, true);
    const size_t ob = bht(d) * d->dv * (d->io == LZ_BF16 ? 2 : 4);
    const char* oc = (const char*)o;
    const char* dc = (const char*)la->dO;
    LZ_REQUIRE(!dc || !nz || dc + ob <= oc || oc + ob <= dc, "dO must not overlap o");
  }
  st = check_ws(d, la ? LZ_WS_HYBRID_FWD_MSE : LZ_WS_HYBRID_FWD, ws, ws_bytes_);
  if (st != LZ_OK) return st;
  const cudaStream_t s = as_stream(stream);
  const bool bf = d->io == LZ_BF16;
  const bool mma = hybrid_uses_mma(d);
  Carver c(ws);
  float* osw = mma ? nullptr : c.take<float>(bht(d) * d->dv);
  void* states16 = fwd_uses_chunks(d) ? c.take<uint16_t>(states16_count(d)) : nullptr;
  const ScanWs scan = fwd_uses_chunks(d) ? carve_scan(c, d) : ScanWs{};
  float* g32 = carve_gates(c, d);
  float* parts = la ? c.take<float>(loss_parts(d)) : nullptr;
  if (states16 && chunk_states && ws_bytes(d, LZ_WS_CHUNK_STATES) > 0) states16 = chunk_states;
  // tensor-core path: the gated state pass (reads k, v, g; writes the chunk
  // states and hT) runs on the side stream while the window forward runs
  // here; gate logits are mapped there too, ahead of it (the window branch
  // does not read the gates; the output pass comes after the join)
  SideStream* side = nullptr;
  const bool fork = mma && fwd_uses_chunks(d) && bht(d) > 0;
  if (fork) {
    cudaError_t e = side_stream(&side);
    if (e == cudaSuccess) e = cudaEventRecord(side->fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side->stream, side->fork, 0);
    if (e != cudaSuccess) return cuda_status(e, "lz_hybrid_fwd (fork)");
  }
  GateIn gi;
  cudaError_t eg = gate_input(d, g, g32, fork ? side->stream : s, gi);
  lz::GlaFwdParams gp = gla_fwd_params(&gi.d, q, k, v, gi.g, h0);
  gp.o = o;
  gp.hT = hT;
  if (fork) {
    gp.states16 = states16;
    gp.delta16 = scan.delta16;
    gp.decay = scan.decay;
    cudaError_t e = eg == cudaSuccess ? lz::launch_gla_states(gp, side->stream) : eg;
    // recorded even after a failed launch: the caller's stream never waits
    // on an unrecorded event
    const cudaError_t ej = cudaEventRecord(side->join, side->stream);
    if (e != cudaSuccess) {
      cudaStreamWaitEvent(s, side->join, 0);
      return cuda_status(e, "lz_hybrid_fwd (gated state pass)");
    }
    if (ej != cudaSuccess) return cuda_status(ej, "lz_hybrid_fwd (join)");
  } else if (eg != cudaSuccess) {
    return cuda_status(eg, "lz_hybrid_fwd (gate logits)");
  }
  lz::SwaFwdParams sp = swa_fwd_params(d, q, k, v, meta_k, meta_v);
  // tensor-core path: bf16 window output into o_swa if requested, else into o
  sp.o = mma ? (o_swa ? o_swa : o) : o_swa;
  sp.o_f32 = osw;
  sp.lse = lse;
  cudaError_t e = swa_forward(sp, bf, s);
  if (e != cudaSuccess) {
    if (side) cudaStreamWaitEvent(s, side->join, 0);
    return cuda_status(e, "lz_hybrid_fwd (window branch)");
  }
  gp.add = osw;
  gp.add16 = mma ? sp.o : nullptr;
  gp.alpha = d->alpha;
  const size_t n = bht(d) * d->dv;
  const float lscale = n > 0 ? (float)(2.0 / (double)n) : 0.f;
  const bool fused = la && loss_fused(d);
  if (fused) {
    gp.target = la->target;
    gp.dO_loss = la->dO;
    gp.loss_scale = lscale;
    gp.loss_part = parts;
  }
  if (side) {  // the state pass ran on the side stream: join it, then the outputs
    e = cudaStreamWaitEvent(s, side->join, 0);
    if (e == cudaSuccess) e = lz::launch_gla_out(gp, s);
  } else {
    e = gla_forward(gp, bf, states16, scan, s);
  }
  if (e != cudaSuccess || !la) return cuda_status(e, name);
  size_t nparts = loss_parts(d);
  if (!fused) {
    e = lz::launch_mse_generic(o, la->target, la->dO, lscale, n, bf, parts, s);
    if (e != cudaSuccess) return cuda_status(e, name);
    nparts = (size_t)lz::mse_generic_parts(n);
  }
  return cuda_status(lz::launch_loss_reduce(parts, nparts, n > 0 ? 1.0 / (double)n : 0.0, la->loss, s),
                     name);
}

lz_status lz_hybrid_fwd(const lz_dims* d, const void* q, const void* k, const void* v,
                        const float* g, const void* meta_k, const void* meta_v,
                        const float* h0, void* o, float* hT, float* lse, void* o_swa,
                        void* chunk_states, void* ws, size_t ws_bytes_, lz_stream stream) {
  return hybrid_fwd_impl("lz_hybrid_fwd", d, q, k, v, g, meta_k, meta_v, h0, o, hT, lse, o_swa,
                         chunk_states, nullptr, ws, ws_bytes_, stream);
}

lz_status lz_hybrid_fwd_mse(const lz_dims* d, const void* q, const void* k, const void* v,
                            const float* g, const void* meta_k, const void* meta_v,
                            const float* h0, const void* target, void* o, float* hT, float* lse,
                            void* o_swa, void* chunk_states, float* loss, void* dO, void* ws,
                            size_t ws_bytes_, lz_stream stream) {
  const LossArgs la{target, loss, dO};
  return hybrid_fwd_impl("lz_hybrid_fwd_mse", d, q, k, v, g, meta_k, meta_v, h0, o, hT, lse, o_swa,
                         chunk_states, &la, ws, ws_bytes_, stream);
}

// The gated backward in two phases: the first (state pass when the forward's
// chunk states are not given; on the tensor-core path also the reverse scan of
// the state gradient) depends only on the inputs, so lz_hybrid_bwd runs it on
// a side stream while the window backward runs; the second computes the
// gradients (and adds them in place to the window branch's).
static cudaError_t gla_bwd_phase1(const lz_dims* d, const void* q, const void* k, const void* v,
                                  const float* g, const float* h0, const void* dO,
                                  const float* dhT, const void* saved_states,
                                  const float* saved_hT, void* dq, void* dk, void* dv, float* dg,
                                  float* dh0, const GlaBwdWs& w, const float* add_dq,
                                  const float* add_dk, const float* add_dv, bool add_in_place,
                                  lz::GlaBwdParams& p, cudaStream_t s) {
  const bool bf = d->io == LZ_BF16;
  const bool mma = bwd_uses_mma(d);
  const void* states16 = w.states16;
  const float* hT = w.hT;
  if (saved_states) {  // the forward's chunk states: no state pass
    states16 = saved_states;
    hT = saved_hT;
  } else {
    lz::GlaFwdParams fp = gla_fwd_params(d, q, k, v, g, h0);
    fp.states = w.states;
    fp.states16 = w.states16;
    fp.hT = w.hT;
    fp.delta16 = w.scan.delta16;
    fp.decay = w.scan.decay;
    cudaError_t e = mma ? lz::launch_gla_states(fp, s) : lz::launch_gla_fwd_simt(fp, bf, s);
    if (e != cudaSuccess) return e;
  }
  p = lz::GlaBwdParams{};
  p.q = q; p.k = k; p.v = v; p.dO = dO; p.dhT = dhT;
  if (d->gate_logits) {
    p.gz = g;
    p.gs = d->gate_scale;
  } else {
    p.g = g;
  }
  p.states = w.states; p.states16 = states16; p.hT = hT;
  p.add_dq = add_dq; p.add_dk = add_dk; p.add_dv = add_dv;
  p.add_in_place = add_in_place;
  p.dq = dq; p.dk = dk; p.dv = dv; p.dg = dg; p.dh0 = dh0;
  p.B = d->B; p.H = d->H; p.T = d->T; p.dkd = d->dk; p.dvd = d->dv;
  if (!mma) return cudaSuccess;
  // two-level: reverse scan of the state gradient
  lz::GlaBwdScanParams sp{};
  sp.q = q; sp.dO = dO; sp.g = p.g; sp.gz = p.gz; sp.gs = p.gs; sp.states16 = states16; sp.dhT = dhT;
  sp.delta16 = w.scan.delta16; sp.decay = w.scan.decay;
  sp.gin16 = w.gin16; sp.gsp = w.gsp; sp.dh0 = dh0;
  sp.B = d->B; sp.H = d->H; sp.T = d->T;
  p.gin16 = w.gin16;
  p.gsp = w.gsp;
  return lz::launch_gla_bwd_scan(sp, s);
}

static cudaError_t gla_bwd_phase2(const lz_dims* d, const lz::GlaBwdParams& p, int* tcflags,
                                  cudaStream_t s) {
  if (!bwd_uses_mma(d)) return lz::launch_gla_bwd_simt(p, d->io == LZ_BF16, s);
  // every chunk at once: tcgen05 for the chunks whose gate factors stay
  // bounded over 128 tokens, then the per-64-row kernel for the others
  if (g_tc_all && tcflags && lz::gla_bwd_tc_supported(p)) {
    cudaError_t e = lz::launch_gla_bwd_tc(p, tcflags, s);
    if (e != cudaSuccess) return e;
    lz::GlaBwdParams q = p;
    q.tc_flags = tcflags;
    return lz::launch_gla_bwd_chunks(q, s);
  }
  return lz::launch_gla_bwd_chunks(p, s);
}

static cudaError_t gla_bwd_launch(const lz_dims* d, const void* q, const void* k, const void* v,
                                  const float* g, const float* h0, const void* dO,
                                  const float* dhT, const void* saved_states,
                                  const float* saved_hT, void* dq, void* dk, void* dv, float* dg,
                                  float* dh0, const GlaBwdWs& w, const float* add_dq,
                                  const float* add_dk, const float* add_dv, bool add_in_place,
                                  cudaStream_t s) {
  lz::GlaBwdParams p;
  cudaError_t e = gla_bwd_phase1(d, q, k, v, g, h0, dO, dhT, saved_states, saved_hT, dq, dk, dv, dg,
                                 dh0, w, add_dq, add_dk, add_dv, add_in_place, p, s);
  if (e != cudaSuccess) return e;
  return gla_bwd_phase2(d, p, w.tcflags, s);
}


lz_status lz_gla_bwd(const lz_dims* d, const void* q, const void* k, const void* v,
                     const float* g, const float* h0, const void* dO, const float* dhT,
                     const void* chunk_states, const float* hT, void* dq, void* dk, void* dv,
                     float* dg, float* dh0, void* ws, size_t ws_bytes_, lz_stream stream) {
  lz_status st = check_dims(d, false);
  if (st != LZ_OK) return st;
  const bool nz = bht(d) > 0;  // empty tensors may have NULL data
  LZ_PTR(q, nz); LZ_PTR(k, nz); LZ_PTR(v, nz); LZ_PTR(g, nz); LZ_PTR(dO, nz);
  LZ_PTR(dq, nz); LZ_PTR(dk, nz); LZ_PTR(dv, nz); LZ_PTR(dg, nz);
  LZ_PTR(h0, false); LZ_PTR(dhT, false); LZ_PTR(dh0, false);
  st = check_saved_states(d, dhT, &chunk_states, hT);
  if (st != LZ_OK) return st;
  st = check_ws(d, LZ_WS_GLA_BWD, ws, ws_bytes_);
  if (st != LZ_OK) return st;
  const cudaStream_t s = as_stream(stream);
  Carver c(ws);
  GlaBwdWs w = carve_gla_bwd(c, d);
  float* g32 = carve_gates(c, d);
  GateIn gi;
  cudaError_t e = gate_input(d, g, g32, s, gi);
  if (e != cudaSuccess) return cuda_status(e, "lz_gla_bwd (gate logits)");
  e = gla_bwd_launch(&gi.d, q, k, v, gi.g, h0, dO, dhT, chunk_states, hT, dq, dk, dv, dg, dh0, w,
                     nullptr, nullptr, nullptr, false, s);
  if (e == cudaSuccess && gi.z) e = lz::launch_gate_dlogit(dg, gi.z, bht(d) * d->dk, d->gate_scale, s);
  return cuda_status(e, "lz_gla_bwd");
}

lz_status lz_swa_meta_bwd(const lz_dims* d, const void* q, const void* k, const void* v,
                          const void* meta_k, const void* meta_v, const float* lse,
                          const void* o, const void* dO, void* dq, void* dk, void* dv,
                          float* dmeta_k, float* dmeta_v, void* ws, size_t ws_bytes_,
                          lz_stream stream) {
  lz_status st = check_dims(d, true);
  if (st != LZ_OK) return st;
  const bool nz = bht(d) > 0;  // empty tensors may have NULL data
  LZ_PTR(q, nz); LZ_PTR(k, nz); LZ_PTR(v, nz); LZ_PTR(lse, nz); LZ_PTR(dO, nz);
  LZ_PTR(dq, nz); LZ_PTR(dk, nz); LZ_PTR(dv, nz);
  LZ_PTR(meta_k, d->M > 0 && d->H > 0); LZ_PTR(meta_v, false); LZ_PTR(o, false);
  LZ_PTR(dmeta_k, false); LZ_PTR(dmeta_v, false);
  st = check_ws(d, LZ_WS_SWA_BWD, ws, ws_bytes_);
  if (st != LZ_OK) return st;
  Carver c(ws);
  SwaBwdWs w = carve_swa_bwd(c, d);
  lz::SwaBwdParams p = swa_bwd_params(d, q, k, v, meta_k, meta_v, lse, o, dO, w);
  p.gscale = 1.f;
  p.dq = dq; p.dk = dk; p.dv = dv;
  p.dmk = dmeta_k; p.dmv = dmeta_v;
  return cuda_status(swa_backward(p, d->io == LZ_BF16, as_stream(stream)), "lz_swa_meta_bwd");
}

lz_status lz_hybrid_bwd(const lz_dims* d, const void* q, const void* k, const void* v,
                        const float* g, const void* meta_k, const void* meta_v,
                        const float* h0, const float* lse, const void* o_swa,
                        const void* chunk_states, const float* hT, const void* dO,
                        const float* dhT,
                        void* dq, void* dk, void* dv, float* dg, float* dh0, float* dmeta_k,
                        float* dmeta_v, float* dalpha, void* ws, size_t ws_bytes_,
                        lz_stream stream) {
  lz_status st = check_dims(d, true);
  if (st != LZ_OK) return st;
  const bool nz = bht(d) > 0;  // empty tensors may have NULL data
  LZ_PTR(q, nz); LZ_PTR(k, nz); LZ_PTR(v, nz); LZ_PTR(g, nz); LZ_PTR(lse, nz);
  LZ_PTR(dO, nz); LZ_PTR(dq, nz); LZ_PTR(dk, nz); LZ_PTR(dv, nz); LZ_PTR(dg, nz);
  LZ_PTR(meta_k, d->M > 0 && d->H > 0); LZ_PTR(meta_v, false); LZ_PTR(h0, false); LZ_PTR(dhT, false);
  LZ_PTR(dh0, false); LZ_PTR(dmeta_k, false); LZ_PTR(dmeta_v, false); LZ_PTR(o_swa, false);
  st = check_saved_states(d, dhT, &chunk_states, hT);
  if (st != LZ_OK) return st;
  if (dalpha && (reinterpret_cast<uintptr_t>(dalpha) & 3u))
    return fail(LZ_ERR_INVALID_ARG, "dalpha must be 4-byte aligned");
  st = check_ws(d, LZ_WS_HYBRID_BWD, ws, ws_bytes_);
  if (st != LZ_OK) return st;
  const cudaStream_t s = as_stream(stream);
  Carver c(ws);
  HybridBwdWs w = carve_hybrid_bwd(c, d);
  float* g32 = carve_gates(c, d);
  GateIn gi;
  const bool mma = hybrid_uses_mma(d);
  lz::SwaBwdParams p = swa_bwd_params(d, q, k, v, meta_k, meta_v, lse, o_swa, dO, w.swa);
  p.gscale = d->alpha;
  // tensor-core path: bf16 window gradients straight into dq, dk, dv; the
  // gated backward then adds its own terms in place
  p.dq = dq; p.dk = dk; p.dv = dv;
  p.dq_f32 = w.dq; p.dk_f32 = w.dk; p.dv_f32 = w.dv;
  p.dmk = dmeta_k; p.dmv = dmeta_v; p.dalpha = dalpha;
  p.ds_tiles = w.ds_tiles; p.ds_meta = w.ds_meta;
  if (!mma || bht(d) == 0) {
    cudaError_t e = gate_input(d, g, g32, s, gi);
    if (e != cudaSuccess) return cuda_status(e, "lz_hybrid_bwd (gate logits)");
    e = swa_backward(p, d->io == LZ_BF16, s);
    if (e != cudaSuccess) return cuda_status(e, "lz_hybrid_bwd (window branch)");
    e = gla_bwd_launch(&gi.d, q, k, v, gi.g, h0, dO, dhT, chunk_states, hT, dq, dk, dv, dg, dh0,
                       w.gla, w.dq, w.dk, w.dv, mma, s);
    if (e == cudaSuccess && gi.z) e = lz::launch_gate_dlogit(dg, gi.z, bht(d) * d->dk, d->gate_scale, s);
    return cuda_status(e, "lz_hybrid_bwd (gated branch)");
  }
  // tensor-core path: the gated backward's first phase (it reads only the
  // inputs and writes only its scratch and dh0) runs on the side stream while
  // the window backward runs here; the second phase adds to the window
  // branch's gradients, so it waits for both
  SideStream* ss = nullptr;
  cudaError_t e = side_stream(&ss);
  if (e != cudaSuccess) return cuda_status(e, "lz_hybrid_bwd (side stream)");
  e = cudaEventRecord(ss->fork, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->stream, ss->fork, 0);
  if (e != cudaSuccess) return cuda_status(e, "lz_hybrid_bwd (fork)");
  lz::GlaBwdParams gp;
  // gate logits are mapped on the side stream, ahead of the gated first phase
  // (the window branch does not read the gates; the second phase comes after
  // the join)
  e = gate_input(d, g, g32, ss->stream, gi);
  if (e == cudaSuccess)
    e = gla_bwd_phase1(&gi.d, q, k, v, gi.g, h0, dO, dhT, chunk_states, hT, dq, dk, dv, dg, dh0,
                       w.gla, w.dq, w.dk, w.dv, mma, gp, ss->stream);
  // the window backward here; its partials' reduction (which needs only the
  // query side) joins the side stream behind the gated first phase, off the
  // path to the per-chunk gradients
  p.query_done = (void*)ss->mid;
  p.defer_reduce = true;
  const cudaError_t esw = e == cudaSuccess ? swa_backward(p, d->io == LZ_BF16, s) : cudaSuccess;
  cudaError_t er = cudaSuccess;
  if (e == cudaSuccess && esw == cudaSuccess) {
    er = cudaStreamWaitEvent(ss->stream, ss->mid, 0);
    if (er == cudaSuccess) er = lz::launch_swa_bwd_mma_reduce(p, ss->stream);
  }
  // the join is recorded even after a failed launch, so that the caller's
  // stream never depends on an unrecorded event
  const cudaError_t ej = cudaEventRecord(ss->join, ss->stream);
  const cudaError_t ew = cudaStreamWaitEvent(s, ss->join, 0);
  if (e != cudaSuccess) return cuda_status(e, "lz_hybrid_bwd (gated branch, first phase)");
  if (esw != cudaSuccess) return cuda_status(esw, "lz_hybrid_bwd (window branch)");
  if (er != cudaSuccess) return cuda_status(er, "lz_hybrid_bwd (window partials)");
  if (ej != cudaSuccess) return cuda_status(ej, "lz_hybrid_bwd (join)");
  if (ew != cudaSuccess) return cuda_status(ew, "lz_hybrid_bwd (join)");
  e = gla_bwd_phase2(&gi.d, gp, w.gla.tcflags, s);
  if (e == cudaSuccess && gi.z) e = lz::launch_gate_dlogit(dg, gi.z, bht(d) * d->dk, d->gate_scale, s);
  return cuda_status(e, "lz_hybrid_bwd (gated branch)");
}

lz_status lz_decode_prefill(int Bd, int H, int T, int dk, int dv, int w, lz_dtype io,
                            const void* k, const void* v, const int64_t* lens, const float* hT,
                            float* state, void* kring, void* vring, int64_t* pos,
                            lz_stream stream) {
  LZ_REQUIRE(Bd >= 0 && H >= 0 && T >= 0, "Bd, H, T must be >= 0 (got %d, %d, %d)", Bd, H, T);
  if (io != LZ_F32 && io != LZ_BF16)
    return fail(LZ_ERR_UNSUPPORTED, "io dtype %d is not LZ_F32 or LZ_BF16", (int)io);
  if (dk != 128 || dv != 128)
    return fail(LZ_ERR_UNSUPPORTED, "decode supports dk = dv = 128 (got %d, %d)", dk, dv);
  if (w < 1 || w > 1024) return fail(LZ_ERR_UNSUPPORTED, "w must be in [1, 1024] (got %d)", w);
  const bool nz = (size_t)Bd * H > 0;
  const bool nzt = nz && T > 0;
  LZ_PTR(k, nzt); LZ_PTR(v, nzt); LZ_PTR(hT, false); LZ_PTR(lens, false);
  LZ_PTR(state, nz); LZ_PTR(kring, nz); LZ_PTR(vring, nz); LZ_PTR(pos, Bd > 0);
  lz::DecodePrefillParams p{};
  p.Bd = Bd; p.H = H; p.T = T; p.w = w;
  p.k = k; p.v = v; p.hT = hT; p.state = state; p.kring = kring; p.vring = vring; p.pos = pos;
  p.lens = lens;
  return cuda_status(lz::launch_decode_prefill(p, io == LZ_BF16, as_stream(stream)),
                     "lz_decode_prefill");
}

lz_status lz_gla_decode_step(int Bd, int H, int dk, int dv, int w, int M, lz_dtype io,
                             float scale, float alpha, float* state, void* kring,
                             void* vring, int64_t* pos, const void* q, const void* k,
                             const void* v, const float* g, const void* meta_k,
                             const void* meta_v, void* o, lz_stream stream) {
  LZ_REQUIRE(Bd >= 0 && H >= 0, "Bd, H must be >= 0 (got %d, %d)", Bd, H);
  if (io != LZ_F32 && io != LZ_BF16)
    return fail(LZ_ERR_UNSUPPORTED, "io dtype %d is not LZ_F32 or LZ_BF16", (int)io);
  if (dk != 128 || dv != 128)
    return fail(LZ_ERR_UNSUPPORTED, "decode supports dk = dv = 128 (got %d, %d)", dk, dv);
  if (H > 32767) return fail(LZ_ERR_UNSUPPORTED, "decode supports H <= 32767 (got %d)", H);
  if (w < 1 || w > 1024) return fail(LZ_ERR_UNSUPPORTED, "w must be in [1, 1024] (got %d)", w);
  if (M < 0 || M > 16) return fail(LZ_ERR_UNSUPPORTED, "M must be in [0, 16] (got %d)", M);
  const bool nz = (size_t)Bd * H > 0;  // empty tensors may have NULL data
  LZ_PTR(state, nz); LZ_PTR(kring, nz); LZ_PTR(vring, nz); LZ_PTR(pos, Bd > 0);
  LZ_PTR(q, nz); LZ_PTR(k, nz); LZ_PTR(v, nz); LZ_PTR(g, nz); LZ_PTR(o, nz);
  LZ_PTR(meta_k, M > 0 && H > 0); LZ_PTR(meta_v, false);
  lz::DecodeParams p{};
  p.Bd = Bd; p.H = H; p.w = w; p.M = M; p.scale = scale; p.alpha = alpha;
  p.state = state; p.kring = kring; p.vring = vring; p.pos = pos;
  p.q = q; p.k = k; p.v = v; p.g = g; p.mk = meta_k; p.mv = M > 0 ? meta_v : nullptr; p.o = o;
  return cuda_status(lz::launch_decode(p, io == LZ_BF16, as_stream(stream)),
                     "lz_gla_decode_step");
}

}  // extern "C"
