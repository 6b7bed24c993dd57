// C ABI of the TTT layer library (include/ttt.h): argument checks, workspace planning and
// the enqueue order of the kernels for the parallel form, the recurrent form and the
// In-Place target. Every contraction goes through run_gemm() / run_swiglu(): bf16 mode
// runs them on the tcgen05 tensor-core engine (a problem it cannot take is refused), fp32
// mode on the fp32 CUDA-core engine.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <initializer_list>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "gemm.h"
#include "ops.h"

namespace ttt {

// Per-device error word written by bounded waits and device-side checks.
static __device__ unsigned g_dev_err_word;

static thread_local char g_msg[512] = "";

void set_error_message(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
}

unsigned* device_error_word() {
  static std::mutex mu;
  static unsigned* addr[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_err_word) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned*>(p);
  }
  return addr[dev];
}

unsigned long long wait_limit_ns() {
  const char* s = getenv("TTT_WAIT_LIMIT_NS");
  if (s && *s) {
    const unsigned long long v = strtoull(s, nullptr, 10);
    if (v >= 100000ull) return v;
  }
  return kDefaultWaitNs;
}

namespace {

// ------------------------------------------------------------------ kernel tracing
struct TraceState {
  std::mutex mu;
  bool on = false;
  int dev = -1;
  int n = 0;
  int cap = 0;
  std::vector<cudaEvent_t> ev;  // 2 per record
  std::vector<const char*> names;
};
TraceState g_trace;

// Brackets one kernel launch with two events on its stream while tracing is enabled.
struct TraceScope {
  int idx = -1;
  cudaStream_t s;
  TraceScope(const char* name, cudaStream_t st) : s(st) {
    if (!g_trace.on) return;
    std::lock_guard<std::mutex> lk(g_trace.mu);
    int d = -1;
    if (!g_trace.on || cudaGetDevice(&d) != cudaSuccess || d != g_trace.dev ||
        g_trace.n >= g_trace.cap)
      return;
    idx = g_trace.n++;
    g_trace.names[idx] = name;
    cudaEventRecord(g_trace.ev[2 * idx], s);
  }
  ~TraceScope() {
    if (idx >= 0) cudaEventRecord(g_trace.ev[2 * idx + 1], s);
  }
};

// "<name>@<engine>" with stable storage, for trace records.
const char* engine_name(const char* name, const char* engine) {
  static std::mutex mu;
  static std::map<std::string, std::string> names;
  std::lock_guard<std::mutex> lk(mu);
  std::string key = std::string(name) + "@" + engine;
  auto it = names.find(key);
  if (it == names.end()) it = names.emplace(key, key).first;
  return it->second.c_str();
}

ttt_status fail(ttt_status st, const char* fmt, ...);

// One contraction. bf16 operands (bf16 mode) run on the tcgen05 tensor-core engine only: a
// problem that engine cannot take is refused with TTT_ERR_UNSUPPORTED, never rerouted.
// fp32 operands (fp32 mode) run on the fp32 CUDA-core engine.
ttt_status run_gemm(const char* name, const GemmProblem& p, cudaStream_t s) {
  if (p.M <= 0 || p.N <= 0 || p.Z0 <= 0 || p.Z1 <= 0) return TTT_OK;
  if (p.A.dtype == DT_BF16 || p.B.dtype == DT_BF16) {
    if (const char* why = umma_unsupported_reason(p))
      return fail(TTT_ERR_UNSUPPORTED, "%s: tensor-core engine: %s (M=%d N=%d K=%d)", name, why,
                  p.M, p.N, p.K);
    TraceScope ts(g_trace.on ? engine_name(name, "tcgen05") : name, s);
    return gemm_umma(p, s, device_error_word(), wait_limit_ns());
  }
  TraceScope ts(g_trace.on ? engine_name(name, "simt") : name, s);
  return gemm_simt(p, s);
}

// A product of the bf16 mode that needs more than bf16 operands: fp32 operands read as tf32
// by the tensor-core engine (never the CUDA cores).
ttt_status run_tf32(const char* name, const GemmProblem& p, cudaStream_t s) {
  if (p.M <= 0 || p.N <= 0 || p.Z0 <= 0 || p.Z1 <= 0) return TTT_OK;
  if (const char* why = umma_tf32_unsupported_reason(p))
    return fail(TTT_ERR_UNSUPPORTED, "%s: tensor-core engine (tf32): %s (M=%d N=%d K=%d)", name,
                why, p.M, p.N, p.K);
  TraceScope ts(g_trace.on ? engine_name(name, "tcgen05") : name, s);
  return gemm_umma_tf32(p, s, device_error_word(), wait_limit_ns());
}

ttt_status run_simt(const char* name, const GemmProblem& p, cudaStream_t s) {
  if (p.M <= 0 || p.N <= 0 || p.Z0 <= 0 || p.Z1 <= 0) return TTT_OK;
  TraceScope ts(g_trace.on ? engine_name(name, "simt") : name, s);
  return gemm_simt(p, s);
}

#define TTT_TRY(expr)                        \
  do {                                       \
    ttt_status st__ = (expr);                \
    if (st__ != TTT_OK) return st__;         \
  } while (0)

#define TTT_CUDA(expr)                                                                    \
  do {                                                                                    \
    cudaError_t e__ = (expr);                                                             \
    if (e__ != cudaSuccess) {                                                             \
      set_error_message("%s failed: %s", #expr, cudaGetErrorString(e__));                 \
      return TTT_ERR_CUDA;                                                                \
    }                                                                                     \
  } while (0)

// One traced kernel launch of ops.h.
#define TTT_OP(name, expr)         \
  do {                             \
    TraceScope ts__((name), s);    \
    TTT_CUDA(expr);                \
  } while (0)

ttt_status fail(ttt_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// ------------------------------------------------------------------ debug checks
// Process-wide TTT_CHECK_* flags (ttt_set_debug_checks), and the guards the calling thread's
// current call carved from its workspace.
std::atomic<int> g_checks{0};
thread_local std::vector<unsigned*> t_guards;

// Bump allocator over the caller's workspace (or a size counter when base is null). With
// TTT_CHECK_GUARDS on, a kGuardBytes guard sits in front of the first region and right
// after the end of every region (16-byte aligned); the guards of a real workspace are
// listed in t_guards.
struct Carve {
  char* base;
  size_t off = 0;
  bool guards;
  explicit Carve(void* b)
      : base(static_cast<char*>(b)), guards((g_checks.load() & TTT_CHECK_GUARDS) != 0) {
    if (guards) guard();
  }
  void guard() {
    off = (off + 15) & ~static_cast<size_t>(15);
    if (base) t_guards.push_back(reinterpret_cast<unsigned*>(base + off));
    off += kGuardBytes;
  }
  void* take(size_t bytes) {
    off = (off + 255) & ~static_cast<size_t>(255);
    void* p = base ? base + off : nullptr;
    off += bytes;
    if (guards) guard();
    return p;
  }
  template <typename T> T* take_n(long long n) { return static_cast<T*>(take(sizeof(T) * (size_t)n)); }
};

// Fills (check = false) or compares (check = true) every guard in t_guards.
ttt_status run_guards(bool check, cudaStream_t s) {
  for (size_t i0 = 0; i0 < t_guards.size(); i0 += kMaxGuards) {
    GuardList g;
    g.n = (int)std::min<size_t>(kMaxGuards, t_guards.size() - i0);
    for (int i = 0; i < g.n; ++i) g.p[i] = t_guards[i0 + i];
    TraceScope ts(check ? "guards_check" : "guards_fill", s);
    const cudaError_t e = check ? guards_check(g, device_error_word(), s) : guards_fill(g, s);
    if (e != cudaSuccess)
      return fail(TTT_ERR_CUDA, "debug guards: %s", cudaGetErrorString(e));
  }
  return TTT_OK;
}

// One output of a call, for the non-finite scan.
struct OutBuf {
  const void* p;
  long long n;
  int dt;
};

// Start of a call's work on `s`: writes the guards of the workspace just planned.
ttt_status checks_begin(cudaStream_t s) {
  if (!(g_checks.load() & TTT_CHECK_GUARDS)) return TTT_OK;
  return run_guards(false, s);
}

// End of a call's work on `s`: compares the guards and scans the outputs.
ttt_status checks_end(cudaStream_t s, std::initializer_list<OutBuf> outs) {
  const int f = g_checks.load();
  if (f & TTT_CHECK_GUARDS) TTT_TRY(run_guards(true, s));
  if (f & TTT_CHECK_FINITE)
    for (const OutBuf& o : outs) {
      if (!o.p || o.n <= 0) continue;
      TraceScope ts("finite_scan", s);
      const cudaError_t e = finite_scan(o.dt, o.p, o.n, device_error_word(), s);
      if (e != cudaSuccess) return fail(TTT_ERR_CUDA, "finite scan: %s", cudaGetErrorString(e));
    }
  return TTT_OK;
}

// A call's body between checks_begin and checks_end; the end runs after a successful body.
template <typename F>
ttt_status with_checks(cudaStream_t s, std::initializer_list<OutBuf> outs, F&& body) {
  TTT_TRY(checks_begin(s));
  TTT_TRY(body());
  return checks_end(s, outs);
}

ttt_status check_desc(const ttt_desc* d, int path) {
  if (!d) return fail(TTT_ERR_INVALID_ARG, "desc is NULL");
  if (d->B < 0 || d->H < 0 || d->N < 0) return fail(TTT_ERR_INVALID_ARG, "B, H, N must be >= 0");
  if (d->h < 1 || d->m < 1 || d->chunk < 1)
    return fail(TTT_ERR_INVALID_ARG, "h, m and chunk must be >= 1");
  if (d->dtype != TTT_DTYPE_FP32 && d->dtype != TTT_DTYPE_BF16)
    return fail(TTT_ERR_INVALID_ARG, "dtype must be TTT_DTYPE_FP32 or TTT_DTYPE_BF16");
  if (d->order != TTT_ORDER_UPDATE_APPLY && d->order != TTT_ORDER_APPLY_UPDATE)
    return fail(TTT_ERR_INVALID_ARG, "order must be UPDATE_APPLY or APPLY_UPDATE");
  if (d->sign != 1 && d->sign != -1) return fail(TTT_ERR_INVALID_ARG, "sign must be +1 or -1");
  if (d->w_in_layout != 0 && d->w_in_layout != 1)
    return fail(TTT_ERR_INVALID_ARG, "w_in_layout must be 0 or 1");
  if (d->w1_layout != 0 && d->w1_layout != 1)
    return fail(TTT_ERR_INVALID_ARG, "w1_layout must be 0 or 1");
  if (path == TTT_PATH_PARALLEL_BWD) {
    if (d->update_mask != 0 || d->renorm != 0 || d->momentum != 0 || d->ns_steps != 0)
      return fail(TTT_ERR_INVALID_ARG,
                  "parallel form: update_mask, renorm, momentum and ns_steps must be 0");
    if (d->w_in_layout != 0 || d->w1_layout != 0)
      return fail(TTT_ERR_UNSUPPORTED, "backward: default weight layouts only");
  } else if (path == TTT_PATH_PARALLEL_MOMENTUM) {
    if (d->update_mask != 0 || d->renorm != 0)
      return fail(TTT_ERR_INVALID_ARG, "parallel form: update_mask and renorm must be 0");
    if (d->momentum != 0 && d->momentum != 1)
      return fail(TTT_ERR_INVALID_ARG, "momentum must be 0 or 1");
    if (d->ns_steps < 0 || d->ns_steps > 8) return fail(TTT_ERR_INVALID_ARG, "ns_steps must be in 0..8");
    if (d->w1_layout != 0)
      return fail(TTT_ERR_UNSUPPORTED, "parallel form with momentum: W1 layout 0 only");
  } else if (path == TTT_PATH_PARALLEL || path == TTT_PATH_LINEAR) {
    if (d->update_mask != 0 || d->renorm != 0 || d->momentum != 0 || d->ns_steps != 0)
      return fail(TTT_ERR_INVALID_ARG,
                  "parallel form: update_mask, renorm, momentum and ns_steps must be 0");
    if (path == TTT_PATH_LINEAR && (d->m != d->h || d->w_in_layout != 0))
      return fail(TTT_ERR_INVALID_ARG, "identity features: m must equal h, w_in_layout 0");
  } else if (path == TTT_PATH_RECURRENT) {
    if (d->update_mask < 1 || d->update_mask > 7)
      return fail(TTT_ERR_INVALID_ARG, "update_mask must be in 1..7");
    if ((d->renorm != 0 && d->renorm != 1) || (d->momentum != 0 && d->momentum != 1))
      return fail(TTT_ERR_INVALID_ARG, "renorm and momentum must be 0 or 1");
    if (d->ns_steps < 0 || d->ns_steps > 8) return fail(TTT_ERR_INVALID_ARG, "ns_steps must be in 0..8");
    if (d->w_in_layout != 0 || d->w1_layout != 0)
      return fail(TTT_ERR_UNSUPPORTED, "recurrent form: only the default weight layouts");
    if (d->h > 1536 || d->m > 1536)
      return fail(TTT_ERR_UNSUPPORTED, "recurrent form: h and m must be <= 1536");
  } else {
    return fail(TTT_ERR_INVALID_ARG, "path must be one of TTT_PATH_*");
  }
  if (d->dtype == TTT_DTYPE_BF16 && (d->h % 8 != 0 || d->m % 8 != 0))
    return fail(TTT_ERR_UNSUPPORTED, "bf16 mode needs h and m to be multiples of 8");
  const long long BH = (long long)d->B * d->H;
  if (BH > 65535) return fail(TTT_ERR_UNSUPPORTED, "B*H must be <= 65535");
  if ((long long)d->N > (1LL << 22)) return fail(TTT_ERR_UNSUPPORTED, "N must be <= 4194304");
  const long long C = (d->N + d->chunk - 1) / d->chunk;
  if (BH * C > 65535 && path != TTT_PATH_RECURRENT)
    return fail(TTT_ERR_UNSUPPORTED, "B*H*ceil(N/chunk) must be <= 65535");
  if ((long long)d->h * d->m > (1LL << 31))
    return fail(TTT_ERR_UNSUPPORTED, "h*m must be <= 2^31");
  return TTT_OK;
}

// ------------------------------------------------------------------ parallel form
struct ParBufs {
  void* Wk;    // [H, 2*mpad, h] blocked [W0^T ; W2^T] operand
  void* phiA;  // phi(K) * eta  [BH, N, m]
  void* phiB;  // phi(Q)        [BH, N, m]
  float* dS;   // [BH, C, m, h]
  void* Sc;    // [BH, C, m, h] state read by each chunk
  float* scan_tmp;   // w1_layout 1: transposed W1 and final state ((H + BH) m h), else null
  float* master;     // sequential schedule: fp32 state per (b, head) (S_final's layout)
  void* shadow;      // sequential schedule: its bf16 copy, the apply GEMMs' operand
};

long long padded_m(int m) { return (m + 127LL) / 128 * 128; }

// The parallel form has two schedules for the same states. The prefix schedule forms every
// chunk's delta at once and scans them, materialising an fp32 delta and a bf16 copy of every
// chunk's state (B H C m h 6 bytes). The sequential schedule keeps one fp32 state per
// (b, head) and, chunk by chunk, applies its bf16 copy and adds the chunk's delta in place
// (an update GEMM with the state as its addend, whose epilogue also refreshes the copy).
// Measured on the In-Place workload (32 states of 11008 x 4096, 8.7 GB materialised): prefix
// 13.3 ms, sequential 14.0 ms per call; the sequential schedule's per-chunk update GEMM is
// bound by its fp32 state traffic. So bf16 mode takes the sequential schedule only when the
// materialised states would exceed 32 GiB, where the prefix schedule's workspace would not
// fit beside the inputs. TTT_SEQUENTIAL=1 or 0 overrides the choice (tests).
bool sequential_schedule(const ttt_desc& d) {
  if (d.dtype != TTT_DTYPE_BF16 || d.N <= 0) return false;
  const long long BH = (long long)d.B * d.H, C = (d.N + d.chunk - 1) / d.chunk;
  const char* e = getenv("TTT_SEQUENTIAL");
  if (e && *e) return e[0] == '1';
  return C > 1 && BH * C * (long long)d.h * d.m * 6 > (32LL << 30);
}

size_t plan_parallel(const ttt_desc& d, void* base, ParBufs& b, bool seq = false) {
  Carve cv(base);
  const size_t os = d.dtype == TTT_DTYPE_BF16 ? 2 : 4;
  const long long BH = (long long)d.B * d.H, C = (d.N + d.chunk - 1) / d.chunk;
  const long long rows = BH * d.N, hm = (long long)d.h * d.m;
  b.Wk = cv.take(os * 2 * padded_m(d.m) * d.h * d.H);
  b.phiA = cv.take(os * rows * d.m);
  b.phiB = cv.take(os * rows * d.m);
  b.master = nullptr;
  b.shadow = nullptr;
  if (seq) {   // sequential schedule: one state per (b, head), no per-chunk states
    b.dS = nullptr;
    b.Sc = nullptr;
    b.scan_tmp = nullptr;
    b.master = cv.take_n<float>(BH * hm);
    b.shadow = cv.take(2 * BH * hm);
    return cv.off;
  }
  b.dS = cv.take_n<float>(BH * C * hm);
  b.Sc = cv.take(os * BH * C * hm);
  b.scan_tmp = d.w1_layout == 1 ? cv.take_n<float>((d.H + BH) * hm) : nullptr;
  return cv.off;
}

// phi(X) for every token of every (b, head): X [B,H,N,h] against the blocked weights of
// its head; writes phi * eta to `scaled` (when eta is set, else phi) and phi to `plain`.
SwigluGemm features_problem(const ttt_desc& d, const void* X, const void* Wk, void* scaled,
                            void* plain, const float* eta) {
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long N = d.N, h = d.h, m = d.m, H = d.H, mp = padded_m(d.m);
  SwigluGemm g;
  GemmProblem& p = g.gemm;
  p.M = d.N; p.N = (int)(2 * mp); p.K = d.h; p.Z0 = d.H; p.Z1 = d.B;
  p.A = {X, ot, false, h, N * h, H * N * h};
  p.B = {Wk, ot, false, h, 2 * mp * h, 0};
  p.C = {scaled, ot, m, N * m, H * N * m};
  g.out2 = plain;
  g.ld2 = m; g.s20 = N * m; g.s21 = H * N * m;
  g.rowscale = eta;
  g.rs0 = N; g.rs1 = H * N;
  g.n_valid = d.m;
  return g;
}

// Feature GEMM with the SwiGLU epilogue: tensor cores for bf16 operands (refused, never
// rerouted, when the engine cannot take the problem), fp32 CUDA cores for fp32 operands.
ttt_status run_swiglu(const char* name, const SwigluGemm& g, cudaStream_t s) {
  const GemmProblem& p = g.gemm;
  if (p.M <= 0 || g.n_valid <= 0 || p.Z0 <= 0 || p.Z1 <= 0) return TTT_OK;
  if (p.A.dtype == DT_BF16 || p.B.dtype == DT_BF16) {
    if (const char* why = umma_swiglu_unsupported_reason(g))
      return fail(TTT_ERR_UNSUPPORTED, "%s: tensor-core engine: %s (M=%d N=%d K=%d)", name, why,
                  p.M, p.N, p.K);
    TraceScope ts(g_trace.on ? engine_name(name, "tcgen05") : name, s);
    return gemm_umma_swiglu(g, s, device_error_word(), wait_limit_ns());
  }
  TraceScope ts(g_trace.on ? engine_name(name, "simt") : name, s);
  return gemm_simt_swiglu(g, s);
}

// Shared by both parallel variants. X_eta: the key-side features times eta, [BH, N, m].
// Delta S_c = sign * X_eta(K_c)^T V_c per (b, head) and chunk, then the prefix scan to the
// state read by each chunk (Sc) and the final state.
ttt_status state_deltas(const ttt_desc& d, const void* X_eta, const void* v, float* dS,
                        cudaStream_t s) {
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long BH = (long long)d.B * d.H, N = d.N, h = d.h, m = d.m, L = d.chunk;
  const long long C = (N + L - 1) / L, Cf = N / L, tail = N - Cf * L, hm = h * m;
  for (int part = 0; part < 2; ++part) {
    const long long nz1 = part == 0 ? Cf : (tail > 0 ? 1 : 0);
    if (nz1 == 0) continue;
    const long long t0 = part == 0 ? 0 : Cf * L;
    GemmProblem p;
    p.M = d.m; p.N = d.h; p.K = (int)(part == 0 ? L : tail); p.Z0 = (int)BH; p.Z1 = (int)nz1;
    p.A = {static_cast<const char*>(X_eta) + t0 * m * dtype_size(ot), ot, true, m, N * m, L * m};
    p.B = {static_cast<const char*>(v) + t0 * h * dtype_size(ot), ot, true, h, N * h, L * h};
    p.C = {dS + (part == 0 ? 0 : Cf * hm), DT_F32, h, C * hm, hm};
    p.alpha = (float)d.sign;
    TTT_TRY(run_gemm("gemm_state_delta", p, s));
  }
  return TTT_OK;
}

// Prefix scan of the chunk deltas to the state read by every chunk (Sc, skipped when null)
// and the final state, from W1 (zero when null) plus n_prior prior states.
ttt_status chunk_states(const ttt_desc& d, const float* dS, const float* W1, float* S_final,
                        void* Sc, float* scan_tmp, cudaStream_t s, const float* prior = nullptr,
                        int n_prior = 0) {
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long BH = (long long)d.B * d.H, C = (d.N + d.chunk - 1) / d.chunk;
  TTT_OP("chunk_scan", chunk_scan(ot, dS, W1, prior, n_prior, Sc, S_final, (int)BH, d.H, (int)C,
                                  d.m, d.h, d.order, d.w1_layout, scan_tmp, s));
  return TTT_OK;
}

ttt_status state_delta_and_scan(const ttt_desc& d, const void* X_eta, const void* v,
                                const float* W1, float* S_final, float* dS, void* Sc,
                                float* scan_tmp, cudaStream_t s) {
  TTT_TRY(state_deltas(d, X_eta, v, dS, s));
  return chunk_states(d, dS, W1, S_final, Sc, scan_tmp, s);
}

// O_c = X_q(Q_c) S_c with X_q the query-side features [BH, N, m].
ttt_status chunk_outputs(const ttt_desc& d, const void* X_q, const void* Sc, void* out,
                         cudaStream_t s) {
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long BH = (long long)d.B * d.H, N = d.N, h = d.h, m = d.m, L = d.chunk;
  const long long C = (N + L - 1) / L, Cf = N / L, tail = N - Cf * L, hm = h * m;
  for (int part = 0; part < 2; ++part) {
    const long long nz1 = part == 0 ? Cf : (tail > 0 ? 1 : 0);
    if (nz1 == 0) continue;
    const long long t0 = part == 0 ? 0 : Cf * L;
    GemmProblem p;
    p.M = (int)(part == 0 ? L : tail); p.N = d.h; p.K = d.m; p.Z0 = (int)BH; p.Z1 = (int)nz1;
    p.A = {static_cast<const char*>(X_q) + t0 * m * dtype_size(ot), ot, false, m, N * m, L * m};
    p.B = {static_cast<const char*>(Sc) + (part == 0 ? 0 : Cf * hm) * dtype_size(ot), ot, true,
           h, C * hm, hm};
    p.C = {static_cast<char*>(out) + t0 * h * dtype_size(ot), ot, h, N * h, L * h};
    TTT_TRY(run_gemm("gemm_output", p, s));
  }
  return TTT_OK;
}

// The chunks' state deltas dS: fused (phi(K) eta kept on chip, one kernel) when the
// problem allows it, else the feature GEMM (phi(K) eta, and phi(Q) when q == k, through
// HBM) followed by the state-delta GEMM.
ttt_status key_side(const ttt_desc& d, const void* k, const void* v, const float* eta,
                    const ParBufs& b, bool shared_qk, cudaStream_t s) {
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  if (!shared_qk && !getenv("TTT_NO_FUSED_DELTA") &&
      fused_delta_supported(ot, d.h, d.m, k, v, eta, b.Wk, b.dS)) {
    TraceScope ts("fused_delta@tcgen05", s);
    return fused_delta(k, v, eta, b.Wk, b.dS, d.B, d.H, d.N, d.h, d.m, d.chunk, d.sign,
                       device_error_word(), wait_limit_ns(), s);
  }
  TTT_TRY(run_swiglu("gemm_features_k",
                     features_problem(d, k, b.Wk, b.phiA, shared_qk ? b.phiB : nullptr, eta),
                     s));
  return state_deltas(d, b.phiA, v, b.dS, s);
}

// The chunks' outputs phi(Q_c) S_c: fused (phi kept on chip) when the problem allows it,
// else (fp32, q == k, other widths, TTT_NO_FUSED_APPLY) the feature GEMM followed by the
// output GEMM.
ttt_status query_side(const ttt_desc& d, const void* q, const ParBufs& b, bool shared_qk,
                      void* out, cudaStream_t s) {
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  if (!shared_qk && !getenv("TTT_NO_FUSED_APPLY") &&
      fused_apply_supported(ot, d.h, d.m, d.chunk, q, b.Wk, b.Sc, out)) {
    // phi(Q) S_c with phi kept on chip
    TraceScope ts("fused_apply@tcgen05", s);
    return fused_apply(q, b.Wk, b.Sc, out, d.B, d.H, d.N, d.h, d.m, d.chunk,
                       device_error_word(), wait_limit_ns(), s);
  }
  if (!shared_qk)
    TTT_TRY(run_swiglu("gemm_features_q",
                       features_problem(d, q, b.Wk, b.phiB, nullptr, nullptr), s));
  return chunk_outputs(d, b.phiB, b.Sc, out, s);
}

// The sequential schedule of the parallel form (see sequential_schedule): features of the
// keys (phi eta) and the queries (phi), the state set to W1 (+ priors), then per chunk the
// apply GEMM O_c = phi(Q_c) S (bf16 copy of S) before or after the update GEMM
// S <- S + sign phi(K_c)^T diag(eta_c) V_c (fp32 S as addend and output, copy refreshed).
ttt_status sequential_impl(const ttt_desc& d, const void* q, const void* k, const void* v,
                           const float* eta, const float* W0, const float* W2, const float* W1,
                           void* out, float* S_final, const ParBufs& b, cudaStream_t s,
                           const float* prior, int n_prior) {
  const int ot = DT_BF16;
  const size_t es = 2;
  const bool shared_qk = (q == k) && out != nullptr;
  const long long BH = (long long)d.B * d.H, N = d.N, h = d.h, m = d.m, L = d.chunk;
  const long long hm = h * m;
  TTT_OP("prep_weights",
         prep_wk_blocked(ot, W0, W2, b.Wk, d.H, d.H, d.h, d.m, d.w_in_layout, s));
  TTT_TRY(run_swiglu("gemm_features_k",
                     features_problem(d, k, b.Wk, b.phiA, shared_qk ? b.phiB : nullptr, eta),
                     s));
  if (out && !shared_qk)
    TTT_TRY(run_swiglu("gemm_features_q",
                       features_problem(d, q, b.Wk, b.phiB, nullptr, nullptr), s));
  float* S = S_final ? S_final : b.master;
  TTT_OP("seq_init", seq_init(W1, prior, n_prior, (int)BH, d.H, hm, S, b.shadow, s));
  const bool t1 = d.w1_layout == 1;   // the state as [h, m] (else [m, h])
  auto apply = [&](long long t0, long long Lc) -> ttt_status {
    GemmProblem p;
    p.M = (int)Lc; p.N = d.h; p.K = d.m; p.Z0 = (int)BH;
    p.A = {static_cast<const char*>(b.phiB) + t0 * m * es, ot, false, m, N * m, 0};
    p.B = t1 ? GemmOperand{b.shadow, ot, false, m, hm, 0}
             : GemmOperand{b.shadow, ot, true, h, hm, 0};
    p.C = {static_cast<char*>(out) + t0 * h * es, ot, h, N * h, 0};
    return run_gemm("gemm_output", p, s);
  };
  auto update = [&](long long t0, long long Lc) -> ttt_status {
    const GemmOperand pe = {static_cast<const char*>(b.phiA) + t0 * m * es, ot, true, m, N * m,
                            0};
    const GemmOperand vv = {static_cast<const char*>(v) + t0 * h * es, ot, true, h, N * h, 0};
    GemmProblem p;
    p.K = (int)Lc; p.Z0 = (int)BH;
    if (t1) {   // S [h, m] += sign V^T (phi eta)
      p.M = d.h; p.N = d.m; p.A = vv; p.B = pe;
      p.C = {S, DT_F32, m, hm, 0};
      p.Cin = {S, m, hm, 0};
    } else {    // S [m, h] += sign (phi eta)^T V
      p.M = d.m; p.N = d.h; p.A = pe; p.B = vv;
      p.C = {S, DT_F32, h, hm, 0};
      p.Cin = {S, h, hm, 0};
    }
    p.C.copy16 = b.shadow;
    p.alpha = (float)d.sign;
    p.beta = 1.0f;
    return run_gemm("gemm_state_update", p, s);
  };
  for (long long t0 = 0; t0 < N; t0 += L) {
    const long long Lc = t0 + L <= N ? L : N - t0;
    if (out && d.order == TTT_ORDER_APPLY_UPDATE) TTT_TRY(apply(t0, Lc));
    TTT_TRY(update(t0, Lc));
    if (out && d.order == TTT_ORDER_UPDATE_APPLY) TTT_TRY(apply(t0, Lc));
  }
  return TTT_OK;
}

// The parallel form; the initial state of (b, head) is W1[head] (zero when W1 is null)
// plus the n_prior states prior[i, b, head]. With out null only the final state is formed
// (no query side, no per-chunk states).
ttt_status parallel_impl(const ttt_desc& d, const void* q, const void* k, const void* v,
                         const float* eta, const float* W0, const float* W2, const float* W1,
                         void* out, float* S_final, const ParBufs& b, cudaStream_t s,
                         const float* prior = nullptr, int n_prior = 0) {
  if (b.master)
    return sequential_impl(d, q, k, v, eta, W0, W2, W1, out, S_final, b, s, prior, n_prior);
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const bool shared_qk = (q == k) && out != nullptr;

  TTT_OP("prep_weights",
         prep_wk_blocked(ot, W0, W2, b.Wk, d.H, d.H, d.h, d.m, d.w_in_layout, s));
  TTT_TRY(key_side(d, k, v, eta, b, shared_qk, s));
  TTT_TRY(chunk_states(d, b.dS, W1, S_final, out ? b.Sc : nullptr, b.scan_tmp, s, prior,
                       n_prior));
  if (!out) return TTT_OK;
  return query_side(d, q, b, shared_qk, out, s);
}

// ------------------------------------------------------------------ identity features
// Variants 3-6 of the simplification ladder: phi = identity, i.e. plain chunked linear
// attention with per-token eta; the state is [h, h].
struct LinBufs {
  void* Keta;  // k * eta  [BH, N, h]
  float* dS;   // [BH, C, h, h]
  void* Sc;    // [BH, C, h, h]
  float* scan_tmp;
};

size_t plan_linear(const ttt_desc& d, void* base, LinBufs& b) {
  Carve cv(base);
  const size_t os = d.dtype == TTT_DTYPE_BF16 ? 2 : 4;
  const long long BH = (long long)d.B * d.H, C = (d.N + d.chunk - 1) / d.chunk;
  const long long hh = (long long)d.h * d.h;
  b.Keta = cv.take(os * BH * d.N * d.h);
  b.dS = cv.take_n<float>(BH * C * hh);
  b.Sc = cv.take(os * BH * C * hh);
  b.scan_tmp = d.w1_layout == 1 ? cv.take_n<float>((d.H + BH) * hh) : nullptr;
  return cv.off;
}

ttt_status linear_impl(const ttt_desc& d, const void* q, const void* k, const void* v,
                       const float* eta, const float* S0, void* out, float* S_final,
                       const LinBufs& b, cudaStream_t s) {
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  TTT_OP("scale_rows", scale_rows(ot, k, eta, b.Keta, (long long)d.B * d.H * d.N, d.h, s));
  TTT_TRY(state_delta_and_scan(d, b.Keta, v, S0, S_final, b.dS, b.Sc, b.scan_tmp, s));
  return chunk_outputs(d, q, b.Sc, out, s);
}

// ------------------------------------------------------------------ Newton-Schulz
// bf16 mode runs Newton-Schulz on the tensor cores at more than bf16 precision: one CTA
// per matrix with split bf16 operands when it fits, else batched GEMMs on tf32 operands;
// fp32 mode uses fp32 CUDA-core products.

// Newton-Schulz scratch of the batched paths (CUDA cores, tf32 GEMMs): X, X2 [problems,
// r, c] (or [c, r]), Ag, Pm [problems, r, r] fp32 and the squared norms. The one-CTA path
// needs none of them.
struct NsScratch {
  float *X = nullptr, *X2 = nullptr, *Ag = nullptr, *Pm = nullptr, *nrm = nullptr;
};

enum NsPath { NS_TENSOR_CTA = 0, NS_TENSOR_GEMM = 1, NS_CUDA_CORES = 2 };

NsPath ns_path(int ot, int R, int C) {
  if (ot == DT_BF16 && ns_mma_supported(R, C)) return NS_TENSOR_CTA;
  if (ot == DT_BF16) return NS_TENSOR_GEMM;
  return NS_CUDA_CORES;
}

NsScratch plan_ns(Carve& cv, int ot, long long problems, int R, int C) {
  NsScratch w;
  const NsPath path = ns_path(ot, R, C);
  if (path == NS_TENSOR_CTA) return w;
  const long long r = R < C ? R : C, c = R < C ? C : R;
  w.X = cv.take_n<float>(problems * r * c);
  w.X2 = cv.take_n<float>(problems * r * c);
  w.Ag = cv.take_n<float>(problems * r * r);
  w.Pm = cv.take_n<float>(problems * r * r);
  w.nrm = cv.take_n<float>(problems);
  return w;
}

// Newton-Schulz (the pages' five-step coefficients, eps 1e-7) in place on the matrices of
// L: tensor cores for bf16 mode when they fit one CTA, else fp32 CUDA-core products (the
// problems of the masked-out parts are computed and not written back).
ttt_status run_ns(int ot, float* U, int Z, const NsLayout& L, int steps, const NsScratch& w,
                  cudaStream_t s, bool nrm_ready = false) {
  const float a3 = 3.4445f, b3 = -4.7750f, c3 = 2.0315f;
  const long long R = L.R[0], Cc = L.C[0];
  if (ot == DT_BF16 && ns_mma_supported((int)R, (int)Cc)) {
    TTT_OP("ns_mma", ns_mma(U, Z, L, steps, 1e-7f, a3, b3, c3, device_error_word(),
                            wait_limit_ns(), s));
    return TTT_OK;
  }
  const long long r = R < Cc ? R : Cc, cc = R < Cc ? Cc : R;
  const int P = Z * L.parts;
  const bool tf32 = ns_path(ot, (int)R, (int)Cc) == NS_TENSOR_GEMM;
  if (tf32) {
    // Each product on the tensor cores with fp32 operands read as tf32 (10-bit mantissa,
    // fp32 accumulation in TMEM). One matrix per entry with R > C ("tall"): the iteration
    // runs on Y = X^T in U's own orientation [c, r], A = Y^T Y (both operands MN-major),
    // Y' = Y P + a Y (P symmetric, so it serves as its own K-major right operand), and the
    // last step writes U. Otherwise on X [r, c] in the wide orientation: A = X X^T (both
    // K-major), X' = P X + a X with X as an MN-major right operand, and the last step writes
    // U when it has that orientation, else a write-back pass transposes the parts back.
    // Either way P = c A A + b A from A (symmetric, K-major both sides).
    const bool tall = L.parts == 1 && R > Cc;
    const bool direct = L.parts == 1 && (L.mask & 1);
    // With one matrix per entry and at least two steps, the first step reads U itself and
    // the normalisation rides on its epilogues: A = s^2 (U^T U) (or U U^T) and the apply
    // s (U P) + a s U, s = 1 / (||U||_F + eps) per entry; no scaled copy is written.
    const bool fold = direct && steps >= 2;
    if (fold) {
      if (!nrm_ready) TTT_OP("ns_sumsq", ns_sumsq(U, Z, L, w.nrm, s));
    } else {
      TTT_OP("ns_normalize", ns_normalize(U, tall ? nullptr : w.X, Z, L, 1e-7f, w.nrm, s,
                                          tall ? w.X : nullptr, nrm_ready));
    }
    auto op = [](const float* ptr, bool mn, long long ld, long long s0) {
      GemmOperand o;
      o.ptr = ptr; o.dtype = DT_F32; o.mn_major = mn; o.ld = ld; o.s0 = s0; o.s1 = 0;
      return o;
    };
    const long long ldx = tall ? r : cc;   // row stride of X (or Y)
    const float* X = fold ? U : w.X;       // this step's input and its entry stride
    long long xs = fold ? L.zstride : r * cc;
    for (int it = 0; it < steps; ++it) {
      const bool scaled = fold && it == 0;
      GemmProblem g1;  // A = X X^T (= Y^T Y)
      g1.M = (int)r; g1.N = (int)r; g1.K = (int)cc; g1.Z0 = P;
      g1.A = op(X, tall, ldx, xs);
      g1.B = op(X, tall, ldx, xs);
      g1.C = {w.Ag, DT_F32, r, r * r, 0};
      if (scaled) { g1.zss = w.nrm; g1.zeps = 1e-7f; g1.zpa = 2; }
      TTT_TRY(run_tf32("ns_gram", g1, s));
      GemmProblem g2;  // P = c A A + b A
      g2.M = (int)r; g2.N = (int)r; g2.K = (int)r; g2.Z0 = P;
      g2.A = op(w.Ag, false, r, r * r);
      g2.B = op(w.Ag, false, r, r * r);
      g2.C = {w.Pm, DT_F32, r, r * r, 0};
      g2.alpha = c3; g2.beta = b3; g2.Cin = {w.Ag, r, r * r, 0};
      TTT_TRY(run_tf32("ns_poly", g2, s));
      const bool last = direct && it == steps - 1;
      float* out = last ? U : (X == w.X ? w.X2 : w.X);
      GemmProblem g3;  // X' = P X + a X (Y' = Y P + a Y)
      g3.K = (int)r; g3.Z0 = P;
      if (tall) {
        g3.M = (int)cc; g3.N = (int)r;
        g3.A = op(X, false, r, xs);
        g3.B = op(w.Pm, false, r, r * r);
      } else {
        g3.M = (int)r; g3.N = (int)cc;
        g3.A = op(w.Pm, false, r, r * r);
        g3.B = op(X, true, cc, xs);
      }
      g3.C = {out, DT_F32, ldx, last ? L.zstride : r * cc, 0};
      g3.alpha = 1.0f; g3.beta = a3; g3.Cin = {X, ldx, xs, 0};
      if (scaled) { g3.zss = w.nrm; g3.zeps = 1e-7f; g3.zpa = 1; g3.zpb = 1; }
      TTT_TRY(run_tf32("ns_apply", g3, s));
      if (last) return TTT_OK;
      X = out;
      xs = r * cc;
    }
    TTT_OP("ns_writeback", ns_writeback(X, U, Z, L, s));
    return TTT_OK;
  }
  TTT_OP("ns_normalize", ns_normalize(U, w.X, Z, L, 1e-7f, w.nrm, s, nullptr, nrm_ready));
  float* X = w.X;
  float* X2 = w.X2;
  for (int it = 0; it < steps; ++it) {
    GemmProblem g1;  // A = X X^T
    g1.M = (int)r; g1.N = (int)r; g1.K = (int)cc; g1.Z0 = P;
    g1.A = {X, DT_F32, false, cc, r * cc, 0};
    g1.B = {X, DT_F32, false, cc, r * cc, 0};
    g1.C = {w.Ag, DT_F32, r, r * r, 0};
    TTT_TRY(run_simt("ns_gram", g1, s));
    GemmProblem g2;  // P = c A A + b A
    g2.M = (int)r; g2.N = (int)r; g2.K = (int)r; g2.Z0 = P;
    g2.A = {w.Ag, DT_F32, false, r, r * r, 0};
    g2.B = {w.Ag, DT_F32, true, r, r * r, 0};
    g2.C = {w.Pm, DT_F32, r, r * r, 0};
    g2.alpha = c3; g2.beta = b3; g2.Cin = {w.Ag, r, r * r, 0};
    TTT_TRY(run_simt("ns_poly", g2, s));
    GemmProblem g3;  // X' = P X + a X
    g3.M = (int)r; g3.N = (int)cc; g3.K = (int)r; g3.Z0 = P;
    g3.A = {w.Pm, DT_F32, false, r, r * r, 0};
    g3.B = {X, DT_F32, true, cc, r * cc, 0};
    g3.C = {X2, DT_F32, cc, r * cc, 0};
    g3.alpha = 1.0f; g3.beta = a3; g3.Cin = {X, cc, r * cc, 0};
    TTT_TRY(run_simt("ns_apply", g3, s));
    float* t = X; X = X2; X2 = t;
  }
  TTT_OP("ns_writeback", ns_writeback(X, U, Z, L, s));
  return TTT_OK;
}

// ------------------------------------------------------------------ momentum + Newton-Schulz
// The parallel form with W1's momentum and orthogonalisation (simplification variant 2).
// With W0, W2 frozen the W1 gradient of chunk c, g_c = -phi(K_c)^T diag(eta_c) V_c, does not
// depend on W1, so for all chunks at once: D_c = sign * phi(K_c)^T diag(eta_c) V_c, the
// momentum scan M_c = alpha_c M_{c-1} + D_c, U_c = NS(M_c) (NS is odd, so the sign and the
// minus of the gradient pass through it), and S_c = W1 + sum_{c' <= c} U_c'.
struct MomBufs {
  ParBufs p;
  NsScratch ns;
};

size_t plan_momentum(const ttt_desc& d, void* base, MomBufs& b) {
  const size_t off = (plan_parallel(d, base, b.p) + 255) & ~static_cast<size_t>(255);
  Carve cv(base ? static_cast<char*>(base) + off : nullptr);
  const long long Z = (long long)d.B * d.H * ((d.N + d.chunk - 1) / d.chunk);
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  b.ns = d.ns_steps > 0 ? plan_ns(cv, ot, Z, d.m, d.h) : NsScratch{};
  return off + cv.off;
}

ttt_status momentum_impl(const ttt_desc& d, const void* q, const void* k, const void* v,
                         const float* eta, const float* alpha, const float* W0, const float* W2,
                         const float* W1, void* out, float* S_final, const MomBufs& mb,
                         cudaStream_t s) {
  const ParBufs& b = mb.p;
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long BH = (long long)d.B * d.H, C = (d.N + d.chunk - 1) / d.chunk;
  const bool shared_qk = (q == k);
  TTT_OP("prep_weights",
         prep_wk_blocked(ot, W0, W2, b.Wk, d.H, d.H, d.h, d.m, d.w_in_layout, s));
  TTT_TRY(key_side(d, k, v, eta, b, shared_qk, s));
  const long long hm = (long long)d.h * d.m;
  // the Frobenius norms of the Newton-Schulz set-up come out of the momentum scan where
  // the batched Newton-Schulz path needs them
  const bool fuse_norms = d.momentum && d.ns_steps > 0 && mb.ns.nrm &&
                          momentum_scan_norms((int)C, hm, b.dS);
  if (d.momentum)
    TTT_OP("momentum_scan", momentum_scan(b.dS, alpha, (int)BH, (int)C, hm, s,
                                          fuse_norms ? mb.ns.nrm : nullptr));
  if (d.ns_steps > 0)
    TTT_TRY(run_ns(ot, b.dS, (int)(BH * C), ns_layout_single(d.m, d.h), d.ns_steps, mb.ns, s,
                   fuse_norms));
  TTT_TRY(chunk_states(d, b.dS, W1, S_final, b.Sc, nullptr, s));
  return query_side(d, q, b, shared_qk, out, s);
}

// ------------------------------------------------------------------ backward
// Gradients of the parallel form (the oracle's la_parallel_backward, in the same order):
// recompute phi(K) eta, phi(K), the chunk states and phi(Q); dS_c = phi(Q_c)^T dO_c; the
// suffix scan gives each delta's gradient G_c and dW1; dphi(Q_c) = dO_c S_c^T,
// dphi(K_c) = sign diag(eta) V_c G_c^T, T_c = phi(K_c) G_c gives dV = sign eta T and
// deta = sign <T, v>; the SwiGLU backward runs as the feature GEMM's gradient epilogue
// (row scale -1: dA = dphi B silu'(A), dB = dphi silu(A)); dX = dA W0^T + dB W2^T and
// dW0 / dW2 = X^T dA / X^T dB per (b, head), summed over the batch.
struct BwdBufs {
  ParBufs p;        // Wk, phiA (phi eta -> dphi(K)), phiB (phi(Q) -> dphi(Q)), dS, Sc
  void* phiK;       // phi(K) [BH, N, m]
  void* G;          // [BH, C, m, h]
  float* R0;        // [BH, m, h]
  void* Ve;         // v * eta [BH, N, h]
  float* T;         // [BH, N, h] fp32 (then dX partials)
  float* neg1;      // [BH * N] = -1
  void* dAB;        // [BH, N, 2m]: dA | dB per token row
  void* Wcat;       // [H, h, 2m]: W0 | W2 operand
  float* dWp;       // [splits, B, H, h, 2m] split-K partials of X^T [dA | dB]
  int splits;
};

// Token splits of the weight-gradient GEMMs (their K is the sequence): enough (b, head,
// split) tiles to fill the SMs twice, splits of at least 512 tokens dividing N.
int bwd_splits(const ttt_desc& d) {
  const long long tiles = (long long)d.B * d.H * ((d.h + 127) / 128) * ((2LL * d.m + 255) / 256);
  int sp = 1;
  while (sp < 64 && d.N % (2 * sp) == 0 && d.N / (2 * sp) >= 512 && tiles * sp < 2 * 148) sp *= 2;
  return sp;
}

size_t plan_backward(const ttt_desc& d, void* base, BwdBufs& b) {
  const size_t off = (plan_parallel(d, base, b.p) + 255) & ~static_cast<size_t>(255);
  Carve cv(base ? static_cast<char*>(base) + off : nullptr);
  const size_t os = d.dtype == TTT_DTYPE_BF16 ? 2 : 4;
  const long long BH = (long long)d.B * d.H, C = (d.N + d.chunk - 1) / d.chunk;
  const long long T = BH * d.N, hm = (long long)d.h * d.m;
  b.phiK = cv.take(os * T * d.m);
  b.G = cv.take(os * BH * C * hm);
  b.R0 = cv.take_n<float>(BH * hm);
  b.Ve = cv.take(os * T * d.h);
  b.T = cv.take_n<float>(T * d.h);
  b.neg1 = cv.take_n<float>(T);
  b.splits = bwd_splits(d);
  b.dAB = cv.take(os * T * 2 * d.m);
  b.Wcat = cv.take(os * d.H * 2 * hm);
  b.dWp = cv.take_n<float>((long long)b.splits * BH * 2 * hm);
  return off + cv.off;
}

// One operand of a per-chunk GEMM: either token rows of [B*H, N, w] sliced to the chunk,
// or the chunk's own matrix of [B*H, C, r, w] (r * w = h * m).
struct ChunkOp {
  const void* ptr;
  int dt;
  bool mn;
  long long w;
  bool tokens;
};

// For every chunk of every (b, head): C_c = alpha * A_c B_c (the chunk-length dimension of
// M, N or K given as -1).
ttt_status chunk_gemm(const char* name, const ttt_desc& d, int M, int Nn, int K, ChunkOp A,
                      ChunkOp B, ChunkOp Cc, float alpha, cudaStream_t s) {
  const long long BH = (long long)d.B * d.H, N = d.N, L = d.chunk, hm = (long long)d.h * d.m;
  const long long C = (N + L - 1) / L, Cf = N / L, tail = N - Cf * L;
  for (int part = 0; part < 2; ++part) {
    const long long nz1 = part == 0 ? Cf : (tail > 0 ? 1 : 0);
    if (nz1 == 0) continue;
    const long long t0 = part == 0 ? 0 : Cf * L, c0 = part == 0 ? 0 : Cf;
    const int Lc = (int)(part == 0 ? L : tail);
    auto op = [&](const ChunkOp& o) {
      const size_t es = dtype_size(o.dt);
      if (o.tokens)
        return GemmOperand{static_cast<const char*>(o.ptr) + t0 * o.w * es, o.dt, o.mn, o.w,
                           N * o.w, L * o.w};
      return GemmOperand{static_cast<const char*>(o.ptr) + c0 * hm * es, o.dt, o.mn, o.w,
                         C * hm, hm};
    };
    GemmProblem p;
    p.M = M < 0 ? Lc : M; p.N = Nn < 0 ? Lc : Nn; p.K = K < 0 ? Lc : K;
    p.Z0 = (int)BH; p.Z1 = (int)nz1;
    p.A = op(A);
    p.B = op(B);
    const GemmOperand c = op(Cc);
    p.C = {const_cast<void*>(c.ptr), c.dtype, c.ld, c.s0, c.s1};
    p.alpha = alpha;
    TTT_TRY(run_gemm(name, p, s));
  }
  return TTT_OK;
}

ttt_status backward_impl(const ttt_desc& d, const void* q, const void* k, const void* v,
                         const float* eta, const float* W0, const float* W2, const float* W1,
                         const void* dO, const float* dS_final, void* dq, void* dk, void* dv,
                         float* deta, float* dW0, float* dW2, float* dW1, const BwdBufs& b,
                         cudaStream_t s) {
  const ParBufs& pb = b.p;
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long BH = (long long)d.B * d.H, N = d.N, h = d.h, m = d.m, H = d.H;
  const long long C = (N + d.chunk - 1) / d.chunk, T = BH * N, hm = h * m;
  const float sg = (float)d.sign;
  // forward recomputation
  TTT_OP("prep_weights",
         prep_wk_blocked(ot, W0, W2, pb.Wk, d.H, d.H, d.h, d.m, d.w_in_layout, s));
  TTT_OP("cast_weights", cat_cols(ot, W0, W2, b.Wcat, H * h, m, s));
  TTT_TRY(run_swiglu("gemm_features_k", features_problem(d, k, pb.Wk, pb.phiA, b.phiK, eta), s));
  TTT_TRY(state_deltas(d, pb.phiA, v, pb.dS, s));
  TTT_TRY(chunk_states(d, pb.dS, W1, nullptr, pb.Sc, nullptr, s));
  TTT_TRY(run_swiglu("gemm_features_q", features_problem(d, q, pb.Wk, pb.phiB, nullptr, nullptr),
                     s));
  // dS_c = phi(Q_c)^T dO_c, then G_c and dW1 per (b, head)
  TTT_TRY(chunk_gemm("gemm_bwd_state", d, d.m, d.h, -1, {pb.phiB, ot, true, m, true},
                     {dO, ot, true, h, true}, {pb.dS, DT_F32, false, h, false}, 1.0f, s));
  TTT_OP("suffix_scan", suffix_scan(ot, pb.dS, dS_final, b.G, b.R0, (int)BH, (int)C, hm,
                                    d.order, s));
  // dphi(Q_c) = dO_c S_c^T (into phiB), dphi(K_c) = sign diag(eta) V_c G_c^T (into phiA)
  TTT_TRY(chunk_gemm("gemm_bwd_dphi_q", d, -1, d.m, d.h, {dO, ot, false, h, true},
                     {pb.Sc, ot, false, h, false}, {pb.phiB, ot, false, m, true}, 1.0f, s));
  TTT_OP("scale_rows", scale_rows(ot, v, eta, b.Ve, T, d.h, s));
  TTT_TRY(chunk_gemm("gemm_bwd_dphi_k", d, -1, d.m, d.h, {b.Ve, ot, false, h, true},
                     {b.G, ot, false, h, false}, {pb.phiA, ot, false, m, true}, sg, s));
  // T_c = phi(K_c) G_c: dV and deta
  TTT_TRY(chunk_gemm("gemm_bwd_t", d, -1, d.h, d.m, {b.phiK, ot, false, m, true},
                     {b.G, ot, true, h, false}, {b.T, DT_F32, false, h, true}, 1.0f, s));
  TTT_OP("row_grads", row_grads(ot, b.T, v, eta, d.sign, dv, deta, T, d.h, s));
  TTT_OP("fill", fill_f32(b.neg1, T, -1.0f, s));
  // SwiGLU backward and input / weight gradients, key side then query side
  const int sp = b.splits;
  const long long Ks = N / sp;
  for (int side = 0; side < 2; ++side) {
    const void* X = side == 0 ? k : q;
    void* dX = side == 0 ? dk : dq;
    // [dA | dB] per token row: the gradient epilogue writes dB (out2) at column m and dA
    // (out3) at column 0 of the same 2m-wide rows
    // (gemm.C names dAB for the epilogue's output layout; that output is skipped)
    SwigluGemm g = features_problem(d, X, pb.Wk, b.dAB, nullptr, b.neg1);
    g.gemm.C.ld = 2 * m; g.gemm.C.s0 = N * 2 * m; g.gemm.C.s1 = H * N * 2 * m;
    g.grad = 1;
    g.skip_out1 = 1;
    g.out2 = static_cast<char*>(b.dAB) + m * dtype_size(ot);
    g.ld2 = 2 * m; g.s20 = N * 2 * m; g.s21 = H * N * 2 * m;
    g.out3 = b.dAB; g.ld3 = 2 * m; g.s30 = N * 2 * m; g.s31 = H * N * 2 * m;
    g.dv = side == 0 ? pb.phiA : pb.phiB;
    g.ldd = m; g.ds0 = N * m; g.ds1 = H * N * m;
    TTT_TRY(run_swiglu(side == 0 ? "gemm_bwd_swiglu_k" : "gemm_bwd_swiglu_q", g, s));
    // dX = [dA | dB] [W0 | W2]^T
    GemmProblem p;
    p.M = d.N; p.N = d.h; p.K = (int)(2 * m); p.Z0 = d.H; p.Z1 = d.B;
    p.A = {b.dAB, ot, false, 2 * m, N * 2 * m, H * N * 2 * m};
    p.B = {b.Wcat, ot, false, 2 * m, 2 * hm, 0};
    p.C = {dX, ot, h, N * h, H * N * h};
    TTT_TRY(run_gemm("gemm_bwd_dx", p, s));
    // X^T [dA | dB] per (b, head) and token split, accumulated over the two sides
    GemmProblem w;
    w.M = d.h; w.N = (int)(2 * m); w.K = (int)Ks; w.Z0 = (int)BH; w.Z1 = sp;
    w.A = {X, ot, true, h, N * h, Ks * h};
    w.B = {b.dAB, ot, true, 2 * m, N * 2 * m, Ks * 2 * m};
    w.C = {b.dWp, DT_F32, 2 * m, 2 * hm, BH * 2 * hm};
    if (side == 1) {
      w.beta = 1.0f;
      w.Cin = {b.dWp, 2 * m, 2 * hm, BH * 2 * hm};
    }
    TTT_TRY(run_gemm("gemm_bwd_dw", w, s));
  }
  TTT_OP("sum_batches", sum_split_cols(b.dWp, sp * d.B, H * h, m, dW0, dW2, s));
  TTT_OP("sum_batches", sum_batches(b.R0, d.B, H * hm, H * hm, dW1, s));
  return TTT_OK;
}

// ------------------------------------------------------------------ recurrent form
struct RecBufs {
  float* W_all;   // fp32 masters [BH][W0^T | W1^T | W2^T], output-major (see ops.h)
  float* M_all;   // momentum, same layout
  float* U;       // update, same layout
  float* tnorm;   // initial column norms per head
  // Three copies of the bf16/fp32 operands, in turn by chunk: the weights after update c
  // are in copy (c + 1) % 3 (the initial weights in copy 0), so the apply reading one copy
  // holds back only the update two chunks later, not the next one.
  void* Wk[3];    // [BH, 2*mpad, h] blocked [W0^T ; W2^T] operand
  void* W1t[3];   // [BH, h, m] W1^T operand
  void* Dv;       // [BH, chunk, m] V W1^T
  void* PE;       // [BH, chunk, 3m]: per token row E0 = d * B * silu'(A) | E2 = d * silu(A) |
                  // P = phi * eta (E0 and E2 side by side: one GEMM gives both gradients)
  float* partials;  // [splits][BH][W0^T | W2^T | W1^T] fp32
  void* phiQ;     // [BH, chunk, m]
  NsScratch ns;   // Newton-Schulz scratch for the 3 matrices of every (b, head)
  int splits;
};

// Token splits of the gradient reductions: the largest power of two that divides the chunk
// length, keeps split lengths a multiple of 64 (and >= 256), keeps the grid of each
// gradient GEMM within one CTA per SM, and keeps all partials within 32 MB. Every split
// writes a full fp32 partial of the three gradients that the reduction reads back, so
// beyond one wave, or once the partials leave L2, more splits cost more traffic than they
// save in GEMM time (measured: 2 splits at lm, 12.6 MB per partial, beat 4 by 12 %; 8 at
// nvs, 2.4 MB per partial, beat 4 by 3 %).
int choose_splits(const ttt_desc& d, long long L) {
  const long long BH = (long long)d.B * d.H;
  // the W0 and W2 gradients are one GEMM of 2m output rows when both are fast
  const bool both = (d.update_mask & TTT_UPDATE_W0) && (d.update_mask & TTT_UPDATE_W2);
  const long long tiles = BH * (((both ? 2 : 1) * d.m + 127) / 128) * ((d.h + 255) / 256);
  const long long partial_bytes = BH * 3LL * d.h * d.m * 4;
  long long best = 1;
  for (long long sp = 2; sp <= 64; sp *= 2) {
    if (L % sp != 0 || (L / sp) % 64 != 0 || L / sp < 256) break;
    if (tiles * sp > 148) break;
    if (sp * partial_bytes > (32LL << 20)) break;
    best = sp;
  }
  return (int)best;
}

// A second stream (and its events) per host thread and device for the recurrent form's
// applies; created on first use. Null if creation fails: the applies then stay on the
// caller's stream.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t gate = nullptr, joined = nullptr, feat = nullptr, g1 = nullptr;
  cudaEvent_t applied[3] = {nullptr, nullptr, nullptr};   // by iteration % 3
  bool ok = false;
};
SideStream* side_stream() {
  constexpr int kMaxDev = 64;
  thread_local SideStream res[kMaxDev];
  thread_local bool tried[kMaxDev] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  SideStream& r = res[dev];
  if (!tried[dev]) {
    tried[dev] = true;
    r.ok = cudaStreamCreateWithFlags(&r.s, cudaStreamNonBlocking) == cudaSuccess &&
           cudaEventCreateWithFlags(&r.gate, cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&r.applied[0], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&r.applied[1], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&r.applied[2], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&r.joined, cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&r.feat, cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&r.g1, cudaEventDisableTiming) == cudaSuccess;
    if (!r.ok) cudaGetLastError();
  }
  return r.ok ? &r : nullptr;
}

size_t plan_recurrent(const ttt_desc& d, void* base, RecBufs& b) {
  Carve cv(base);
  const size_t os = d.dtype == TTT_DTYPE_BF16 ? 2 : 4;
  const long long BH = (long long)d.B * d.H, hm = (long long)d.h * d.m, L = d.chunk;
  const long long rows = BH * L;
  b.splits = choose_splits(d, L);
  b.W_all = cv.take_n<float>(BH * 3 * hm);
  b.M_all = d.momentum ? cv.take_n<float>(BH * 3 * hm) : nullptr;
  b.U = cv.take_n<float>(BH * 3 * hm);
  b.tnorm = cv.take_n<float>((long long)d.H * (2 * d.m + d.h));
  for (int i = 0; i < 3; ++i) {
    b.Wk[i] = cv.take(os * BH * 2 * padded_m(d.m) * d.h);
    b.W1t[i] = cv.take(os * BH * hm);
  }
  b.Dv = cv.take(os * rows * d.m);
  b.PE = cv.take(os * rows * 3 * d.m);
  b.partials = cv.take_n<float>((long long)b.splits * BH * 3 * hm);
  b.phiQ = cv.take(os * rows * d.m);
  b.ns = d.ns_steps > 0 ? plan_ns(cv, d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32, BH * 3,
                                   d.h, d.m)
                        : NsScratch{};
  return cv.off;
}

// Features of tokens [t0, t0 + Lc) of every (b, head) against that (b, head)'s own blocked
// weights; rows of the outputs are chunk-local ([BH, chunk, m]).
SwigluGemm rec_features(const ttt_desc& d, const void* X, const void* Wk, long long t0,
                        long long Lc, void* out) {
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long BH = (long long)d.B * d.H, N = d.N, h = d.h, m = d.m, mp = padded_m(d.m);
  const long long L = d.chunk;
  SwigluGemm g;
  GemmProblem& p = g.gemm;
  p.M = (int)Lc; p.N = (int)(2 * mp); p.K = d.h; p.Z0 = (int)BH; p.Z1 = 1;
  p.A = {static_cast<const char*>(X) + t0 * h * dtype_size(ot), ot, false, h, N * h, 0};
  p.B = {Wk, ot, false, h, 2 * mp * h, 0};
  p.C = {out, ot, m, L * m, 0};
  g.n_valid = d.m;
  return g;
}

// Outputs of tokens [t0, t0 + Lc) with the weights in operand copy `bi`.
ttt_status rec_apply(const ttt_desc& d, const void* q, void* out, long long t0, long long Lc,
                     const RecBufs& b, int bi, cudaStream_t s) {
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const size_t es = dtype_size(ot);
  const long long BH = (long long)d.B * d.H, N = d.N, h = d.h, m = d.m, L = d.chunk;
  TTT_TRY(run_swiglu("gemm_features_q", rec_features(d, q, b.Wk[bi], t0, Lc, b.phiQ), s));
  GemmProblem o;
  o.M = (int)Lc; o.N = d.h; o.K = d.m; o.Z0 = (int)BH; o.Z1 = 1;
  o.A = {b.phiQ, ot, false, m, L * m, 0};
  o.B = {b.W1t[bi], ot, false, m, m * h, 0};   // W1^T rows: K-major
  o.C = {static_cast<char*>(out) + t0 * h * es, ot, h, N * h, 0};
  return run_gemm("gemm_output", o, s);
}

// One gradient step on chunk c (tokens [t0, t0 + Lc)) from the weights in operand copy
// `bin`; the updated operands are written to copy `bout`. With a second stream `side`, the
// W1 gradient runs there alongside the W0 / W2 gradients, and `side->gate` is recorded on
// `s` where work on the second stream may best start alongside the update: just before the
// Newton-Schulz kernel when that kernel runs one CTA per matrix (it leaves most SMs idle),
// else at the start of the update.
ttt_status rec_update(const ttt_desc& d, const void* k, const void* v, const float* eta,
                      const float* alpha, int c, long long t0, long long Lc, const RecBufs& b,
                      int bin, int bout, SideStream* side, cudaStream_t s) {
  const cudaEvent_t gate = side ? side->gate : nullptr;
  const int ot_ = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const bool ns_gate = d.ns_steps > 0 && ns_path(ot_, d.h, d.m) == NS_TENSOR_CTA;
  if (gate && !ns_gate) TTT_CUDA(cudaEventRecord(gate, s));
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const size_t es = dtype_size(ot);
  const long long BH = (long long)d.B * d.H, N = d.N, h = d.h, m = d.m, hm = h * m;
  const long long L = d.chunk;
  const int mask = d.update_mask;
  const bool need_in = (mask & (TTT_UPDATE_W0 | TTT_UPDATE_W2)) != 0;
  const long long C = (N + d.chunk - 1) / d.chunk;
  if (need_in) {  // Dv = V_c W1^T
    GemmProblem g;
    g.M = (int)Lc; g.N = d.m; g.K = d.h; g.Z0 = (int)BH; g.Z1 = 1;
    g.A = {static_cast<const char*>(v) + t0 * h * es, ot, false, h, N * h, 0};
    g.B = {b.W1t[bin], ot, true, m, m * h, 0};   // W1^T rows: MN-major
    g.C = {b.Dv, ot, m, L * m, 0};
    TTT_TRY(run_gemm("gemm_v_w1t", g, s));
  }
  // [A | B] = K_c [W0 | W2] -> P = phi eta (and E2, E0 for the input-side matrices), all
  // three in the rows of PE
  char* PE = static_cast<char*>(b.PE);
  SwigluGemm f = rec_features(d, k, b.Wk[bin], t0, Lc, PE + 2 * m * es);
  f.gemm.C.ld = 3 * m;
  f.gemm.C.s0 = L * 3 * m;
  f.rowscale = eta + t0;
  f.rs0 = N;
  f.rs1 = 0;
  if (need_in) {
    f.grad = 1;
    f.out2 = (mask & TTT_UPDATE_W2) ? PE + m * es : nullptr;
    f.ld2 = 3 * m; f.s20 = L * 3 * m; f.s21 = 0;
    f.out3 = (mask & TTT_UPDATE_W0) ? PE : nullptr;
    f.ld3 = 3 * m; f.s30 = L * 3 * m; f.s31 = 0;
    f.dv = b.Dv;
    f.ldd = m; f.ds0 = L * m; f.ds1 = 0;
  }
  TTT_TRY(run_swiglu("gemm_features_k", f, s));
  // Split-K gradient reductions over the chunk's tokens.
  const int sp = (Lc == d.chunk) ? b.splits : 1;
  const long long Ks = Lc / sp;
  const long long tot = BH * 3 * hm;
  const bool g1_side = side && (mask & TTT_UPDATE_W1) &&
                       (mask & (TTT_UPDATE_W0 | TTT_UPDATE_W2));
  const cudaStream_t s1 = g1_side ? side->s : s;
  if (g1_side) {
    TTT_CUDA(cudaEventRecord(side->feat, s));
    TTT_CUDA(cudaStreamWaitEvent(s1, side->feat, 0));
  }
  if (mask & TTT_UPDATE_W1) {  // dW1^T = -V^T (phi eta), output-major [h, m]
    GemmProblem g;
    g.M = d.h; g.N = d.m; g.K = (int)Ks; g.Z0 = (int)BH; g.Z1 = sp;
    g.A = {static_cast<const char*>(v) + t0 * h * es, ot, true, h, N * h, Ks * h};
    g.B = {PE + 2 * m * es, ot, true, 3 * m, L * 3 * m, Ks * 3 * m};
    g.C = {b.partials + 2 * hm, DT_F32, m, 3 * hm, tot};
    g.alpha = -1.0f;
    TTT_TRY(run_gemm("gemm_grad_w1", g, s1));
  }
  if (g1_side) TTT_CUDA(cudaEventRecord(side->g1, s1));
  {  // [dW0^T ; dW2^T] = [E0 | E2]^T K: [2m, h] in one GEMM (or one of them alone)
    const bool g0 = (mask & TTT_UPDATE_W0) != 0, g2 = (mask & TTT_UPDATE_W2) != 0;
    if (g0 || g2) {
      GemmProblem g;
      g.M = (g0 && g2) ? 2 * d.m : d.m; g.N = d.h; g.K = (int)Ks; g.Z0 = (int)BH; g.Z1 = sp;
      g.A = {PE + (g0 ? 0 : m * es), ot, true, 3 * m, L * 3 * m, Ks * 3 * m};
      g.B = {static_cast<const char*>(k) + t0 * h * es, ot, true, h, N * h, Ks * h};
      g.C = {b.partials + (g0 ? 0 : hm), DT_F32, h, 3 * hm, tot};
      TTT_TRY(run_gemm((g0 && g2) ? "gemm_grad_w02" : g0 ? "gemm_grad_w0" : "gemm_grad_w2", g,
                       s));
    }
  }
  if (g1_side) TTT_CUDA(cudaStreamWaitEvent(s, side->g1, 0));
  if (d.ns_steps > 0) {
    // the update is orthogonalised: sum the splits (and the momentum) into U first
    TTT_OP("reduce_momentum", rec_reduce(b.partials, sp, b.U, d.momentum ? b.M_all : nullptr,
                                        alpha, (int)C, c, (int)BH, d.h, d.m, mask, s));
    if (gate && ns_gate) TTT_CUDA(cudaEventRecord(gate, s));
    TTT_TRY(run_ns(ot, b.U, (int)BH, ns_layout_weights(d.h, d.m, mask), d.ns_steps,
                   b.ns, s));
    TTT_OP("step_renorm", rec_step(b.W_all, b.U, nullptr, 0, nullptr, nullptr, (int)C, c,
                                    b.tnorm, (int)BH, d.H, d.h, d.m, mask, d.sign, d.renorm,
                                    b.Wk[bout], b.W1t[bout], ot, s));
  } else {
    // the split sum and the momentum folded into the step
    TTT_OP("step_renorm", rec_step(b.W_all, nullptr, b.partials, sp,
                                    d.momentum ? b.M_all : nullptr, alpha, (int)C, c, b.tnorm,
                                    (int)BH, d.H, d.h, d.m, mask, d.sign, d.renorm, b.Wk[bout],
                                    b.W1t[bout], ot, s));
  }
  return TTT_OK;
}

ttt_status check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return TTT_OK;
  if (!ws) return fail(TTT_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
  if (reinterpret_cast<uintptr_t>(ws) & 255)
    return fail(TTT_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (have < need)
    return fail(TTT_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", have, need);
  return TTT_OK;
}

}  // namespace
}  // namespace ttt

namespace ttt {
namespace {
// The last successful state-only shard call on this thread, whose workspace still holds the
// blocked weights and the chunk deltas for ttt_la_parallel_fwd_shard_outputs.
struct ShardMark {
  bool valid = false;
  ttt_desc d{};
  void* ws = nullptr;
  size_t bytes = 0;
};
thread_local ShardMark t_shard_mark;
}  // namespace
}  // namespace ttt

using namespace ttt;

extern "C" {

size_t ttt_workspace_bytes(const ttt_desc* desc, int32_t path) {
  if (check_desc(desc, path) != TTT_OK) return 0;
  if (path == TTT_PATH_PARALLEL) {
    ParBufs b;
    return plan_parallel(*desc, nullptr, b, sequential_schedule(*desc));
  }
  if (path == TTT_PATH_LINEAR) {
    LinBufs b;
    return plan_linear(*desc, nullptr, b);
  }
  if (path == TTT_PATH_PARALLEL_MOMENTUM) {
    MomBufs b;
    return plan_momentum(*desc, nullptr, b);
  }
  if (path == TTT_PATH_PARALLEL_BWD) {
    BwdBufs b;
    return plan_backward(*desc, nullptr, b);
  }
  RecBufs b;
  return plan_recurrent(*desc, nullptr, b);
}

ttt_status ttt_la_parallel_fwd(const ttt_desc* desc, const void* q, const void* k, const void* v,
                               const float* eta, const float* W0, const float* W2,
                               const float* W1, void* out, float* S_final, void* workspace,
                               size_t workspace_bytes, ttt_stream_t stream) {
  TTT_TRY(check_desc(desc, TTT_PATH_PARALLEL));
  const ttt_desc& d = *desc;
  const long long BH = (long long)d.B * d.H;
  if (BH == 0) return TTT_OK;
  if (!W0 || !W2 || !W1) return fail(TTT_ERR_INVALID_ARG, "W0, W2 and W1 must not be NULL");
  if (d.N > 0) {
    if (!q || !k || !v || !eta || !out)
      return fail(TTT_ERR_INVALID_ARG, "q, k, v, eta and out must not be NULL");
    if (!al16(q) || !al16(k) || !al16(v) || !al16(out) || !al16(W0) || !al16(W2) || !al16(W1))
      return fail(TTT_ERR_INVALID_ARG, "q, k, v, out and the weights must be 16-byte aligned");
  }
  ParBufs b;
  const bool seq = sequential_schedule(d);
  const size_t need = plan_parallel(d, nullptr, b, seq);
  TTT_TRY(check_ws(workspace, workspace_bytes, need));
  t_guards.clear();
  plan_parallel(d, workspace, b, seq);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long hm = (long long)d.h * d.m;
  return with_checks(s, {{out, BH * d.N * d.h, ot}, {S_final, BH * hm, DT_F32}},
                     [&]() -> ttt_status {
    if (d.N == 0) {
      if (S_final)
        TTT_OP("chunk_scan", chunk_scan(DT_F32, b.dS, W1, nullptr, 0, b.Sc, S_final, (int)BH, d.H,
                                        0, d.m, d.h, d.order, d.w1_layout, nullptr, s));
      return TTT_OK;
    }
    return parallel_impl(d, q, k, v, eta, W0, W2, W1, out, S_final, b, s);
  });
}

ttt_status ttt_la_parallel_fwd_shard(const ttt_desc* desc, const void* q, const void* k,
                                     const void* v, const float* eta, const float* W0,
                                     const float* W2, const float* W1, const float* prior,
                                     int32_t n_prior, void* out, float* S_final, void* workspace,
                                     size_t workspace_bytes, ttt_stream_t stream) {
  t_shard_mark.valid = false;
  TTT_TRY(check_desc(desc, TTT_PATH_PARALLEL));
  const ttt_desc& d = *desc;
  const long long BH = (long long)d.B * d.H;
  if (BH == 0) return TTT_OK;
  if (!W0 || !W2) return fail(TTT_ERR_INVALID_ARG, "W0 and W2 must not be NULL");
  if (n_prior < 0 || n_prior > 4096) return fail(TTT_ERR_INVALID_ARG, "n_prior must be in 0..4096");
  if (n_prior > 0 && (!prior || !al16(prior)))
    return fail(TTT_ERR_INVALID_ARG, "prior must be a 16-byte aligned pointer when n_prior > 0");
  if (!out && !S_final) return fail(TTT_ERR_INVALID_ARG, "out and S_final are both NULL");
  if ((W1 && !al16(W1)) || !al16(W0) || !al16(W2))
    return fail(TTT_ERR_INVALID_ARG, "the weights must be 16-byte aligned");
  if (d.N > 0) {
    if (!q || !k || !v || !eta)
      return fail(TTT_ERR_INVALID_ARG, "q, k, v and eta must not be NULL");
    if (!al16(q) || !al16(k) || !al16(v) || (out && !al16(out)))
      return fail(TTT_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
  }
  ParBufs b;
  const bool seq = sequential_schedule(d);
  const size_t need = plan_parallel(d, nullptr, b, seq);
  TTT_TRY(check_ws(workspace, workspace_bytes, need));
  t_guards.clear();
  plan_parallel(d, workspace, b, seq);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long hm = (long long)d.h * d.m;
  return with_checks(s, {{out, BH * d.N * d.h, ot}, {S_final, BH * hm, DT_F32}},
                     [&]() -> ttt_status {
    if (d.N == 0) {
      if (S_final)
        TTT_OP("chunk_scan", chunk_scan(DT_F32, b.dS, W1, prior, n_prior, nullptr, S_final,
                                        (int)BH, d.H, 0, d.m, d.h, d.order, d.w1_layout,
                                        b.scan_tmp, s));
      return TTT_OK;
    }
    const ttt_status st =
        parallel_impl(d, q, k, v, eta, W0, W2, W1, out, S_final, b, s, prior, n_prior);
    if (st == TTT_OK && !out && !seq) {
      // the blocked weights and every chunk's delta stay in the workspace for an outputs pass
      t_shard_mark.valid = true;
      t_shard_mark.d = d;
      t_shard_mark.ws = workspace;
      t_shard_mark.bytes = workspace_bytes;
    }
    return st;
  });
}

ttt_status ttt_la_parallel_fwd_shard_outputs(const ttt_desc* desc, const void* q,
                                             const float* W1, const float* prior,
                                             int32_t n_prior, void* out, float* S_final,
                                             void* workspace, size_t workspace_bytes,
                                             ttt_stream_t stream) {
  TTT_TRY(check_desc(desc, TTT_PATH_PARALLEL));
  const ttt_desc& d = *desc;
  const ShardMark mk = t_shard_mark;
  t_shard_mark.valid = false;
  if (sequential_schedule(d))
    return fail(TTT_ERR_UNSUPPORTED, "the sequential schedule keeps no chunk deltas: run the "
                                     "shard call again with out");
  if (!mk.valid || mk.ws != workspace || mk.bytes != workspace_bytes ||
      std::memcmp(&mk.d, &d, sizeof(ttt_desc)) != 0)
    return fail(TTT_ERR_INVALID_ARG, "an outputs pass must follow, on this thread, a state-only "
                                     "shard call with the same descriptor and workspace");
  const long long BH = (long long)d.B * d.H;
  if (BH == 0 || d.N == 0) return TTT_OK;
  if (!q || !out) return fail(TTT_ERR_INVALID_ARG, "q and out must not be NULL");
  if (!al16(q) || !al16(out) || (W1 && !al16(W1)))
    return fail(TTT_ERR_INVALID_ARG, "q, out and W1 must be 16-byte aligned");
  if (n_prior < 0 || n_prior > 4096) return fail(TTT_ERR_INVALID_ARG, "n_prior must be in 0..4096");
  if (n_prior > 0 && (!prior || !al16(prior)))
    return fail(TTT_ERR_INVALID_ARG, "prior must be a 16-byte aligned pointer when n_prior > 0");
  ParBufs b;
  plan_parallel(d, workspace, b, false);
  t_guards.clear();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long hm = (long long)d.h * d.m;
  return with_checks(s, {{out, BH * d.N * d.h, ot}, {S_final, BH * hm, DT_F32}},
                     [&]() -> ttt_status {
    TTT_TRY(chunk_states(d, b.dS, W1, S_final, b.Sc, b.scan_tmp, s, prior, n_prior));
    return query_side(d, q, b, false, out, s);
  });
}

ttt_status ttt_linear_attn_fwd(const ttt_desc* desc, const void* q, const void* k, const void* v,
                               const float* eta, const float* S0, void* out, float* S_final,
                               void* workspace, size_t workspace_bytes, ttt_stream_t stream) {
  TTT_TRY(check_desc(desc, TTT_PATH_LINEAR));
  const ttt_desc& d = *desc;
  const long long BH = (long long)d.B * d.H;
  if (BH == 0) return TTT_OK;
  if (!S0) return fail(TTT_ERR_INVALID_ARG, "S0 must not be NULL");
  if (d.N > 0) {
    if (!q || !k || !v || !eta || !out)
      return fail(TTT_ERR_INVALID_ARG, "q, k, v, eta and out must not be NULL");
    if (!al16(q) || !al16(k) || !al16(v) || !al16(out) || !al16(S0))
      return fail(TTT_ERR_INVALID_ARG, "q, k, v, out and S0 must be 16-byte aligned");
  }
  LinBufs b;
  const size_t need = plan_linear(d, nullptr, b);
  TTT_TRY(check_ws(workspace, workspace_bytes, need));
  t_guards.clear();
  plan_linear(d, workspace, b);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  return with_checks(s, {{out, BH * d.N * d.h, ot}, {S_final, BH * d.h * d.h, DT_F32}},
                     [&]() -> ttt_status {
    if (d.N == 0) {
      if (S_final)
        TTT_OP("chunk_scan", chunk_scan(DT_F32, b.dS, S0, nullptr, 0, b.Sc, S_final, (int)BH, d.H,
                                        0, d.h, d.h, d.order, d.w1_layout, nullptr, s));
      return TTT_OK;
    }
    return linear_impl(d, q, k, v, eta, S0, out, S_final, b, s);
  });
}

ttt_status ttt_la_parallel_momentum_fwd(const ttt_desc* desc, const void* q, const void* k,
                                        const void* v, const float* eta, const float* alpha,
                                        const float* W0, const float* W2, const float* W1,
                                        void* out, float* S_final, void* workspace,
                                        size_t workspace_bytes, ttt_stream_t stream) {
  TTT_TRY(check_desc(desc, TTT_PATH_PARALLEL_MOMENTUM));
  const ttt_desc& d = *desc;
  const long long BH = (long long)d.B * d.H;
  if (BH == 0) return TTT_OK;
  if (!W0 || !W2 || !W1) return fail(TTT_ERR_INVALID_ARG, "W0, W2 and W1 must not be NULL");
  if (d.momentum && d.N > 0 && !alpha)
    return fail(TTT_ERR_INVALID_ARG, "momentum needs alpha");
  if (d.N > 0) {
    if (!q || !k || !v || !eta || !out)
      return fail(TTT_ERR_INVALID_ARG, "q, k, v, eta and out must not be NULL");
    if (!al16(q) || !al16(k) || !al16(v) || !al16(out) || !al16(W0) || !al16(W2) || !al16(W1))
      return fail(TTT_ERR_INVALID_ARG, "q, k, v, out and the weights must be 16-byte aligned");
  }
  MomBufs b;
  const size_t need = plan_momentum(d, nullptr, b);
  TTT_TRY(check_ws(workspace, workspace_bytes, need));
  t_guards.clear();
  plan_momentum(d, workspace, b);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long hm = (long long)d.h * d.m;
  return with_checks(s, {{out, BH * d.N * d.h, ot}, {S_final, BH * hm, DT_F32}},
                     [&]() -> ttt_status {
    if (d.N == 0) {
      if (S_final)
        TTT_OP("chunk_scan", chunk_scan(DT_F32, b.p.dS, W1, nullptr, 0, b.p.Sc, S_final, (int)BH,
                                        d.H, 0, d.m, d.h, d.order, d.w1_layout, nullptr, s));
      return TTT_OK;
    }
    return momentum_impl(d, q, k, v, eta, alpha, W0, W2, W1, out, S_final, b, s);
  });
}

ttt_status ttt_la_parallel_bwd(const ttt_desc* desc, const void* q, const void* k, const void* v,
                               const float* eta, const float* W0, const float* W2,
                               const float* W1, const void* dout, const float* dS_final,
                               void* dq, void* dk, void* dv, float* deta, float* dW0,
                               float* dW2, float* dW1, void* workspace, size_t workspace_bytes,
                               ttt_stream_t stream) {
  TTT_TRY(check_desc(desc, TTT_PATH_PARALLEL_BWD));
  const ttt_desc& d = *desc;
  const long long BH = (long long)d.B * d.H;
  if (BH == 0) return TTT_OK;
  if (!W0 || !W2 || !W1 || !dW0 || !dW2 || !dW1)
    return fail(TTT_ERR_INVALID_ARG, "weights and weight gradients must not be NULL");
  if (d.N > 0) {
    if (!q || !k || !v || !eta || !dout || !dq || !dk || !dv || !deta)
      return fail(TTT_ERR_INVALID_ARG, "inputs, dout and input gradients must not be NULL");
    if (q == k || dq == dk)
      return fail(TTT_ERR_INVALID_ARG, "backward: q and k (and dq, dk) must be distinct");
    const void* ptrs[] = {q, k, v, dout, dq, dk, dv, W0, W2, W1, eta, deta};
    for (const void* p : ptrs)
      if (!al16(p)) return fail(TTT_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  }
  BwdBufs b;
  const size_t need = plan_backward(d, nullptr, b);
  TTT_TRY(check_ws(workspace, workspace_bytes, need));
  t_guards.clear();
  plan_backward(d, workspace, b);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long hm = (long long)d.h * d.m;
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  const long long T = BH * d.N;
  return with_checks(s, {{dq, T * d.h, ot}, {dk, T * d.h, ot}, {dv, T * d.h, ot},
                         {deta, T, DT_F32}, {dW0, d.H * hm, DT_F32}, {dW2, d.H * hm, DT_F32},
                         {dW1, d.H * hm, DT_F32}},
                     [&]() -> ttt_status {
    if (d.N == 0) {   // no outputs: dW1 = sum over the batch of dS_final, the rest zero
      TTT_OP("fill", fill_f32(dW0, d.H * hm, 0.0f, s));
      TTT_OP("fill", fill_f32(dW2, d.H * hm, 0.0f, s));
      if (dS_final)
        TTT_OP("sum_batches", sum_batches(dS_final, d.B, d.H * hm, d.H * hm, dW1, s));
      else
        TTT_OP("fill", fill_f32(dW1, d.H * hm, 0.0f, s));
      return TTT_OK;
    }
    return backward_impl(d, q, k, v, eta, W0, W2, W1, dout, dS_final, dq, dk, dv, deta, dW0,
                         dW2, dW1, b, s);
  });
}

ttt_status ttt_lact_recurrent_fwd(const ttt_desc* desc, const void* q, const void* k,
                                  const void* v, const float* eta, const float* alpha,
                                  const float* W0, const float* W2, const float* W1, void* out,
                                  float* W0_out, float* W2_out, float* W1_out, float* M_io,
                                  void* workspace, size_t workspace_bytes, ttt_stream_t stream) {
  TTT_TRY(check_desc(desc, TTT_PATH_RECURRENT));
  const ttt_desc& d = *desc;
  const long long BH = (long long)d.B * d.H;
  if (BH == 0) return TTT_OK;
  if (!W0 || !W2 || !W1) return fail(TTT_ERR_INVALID_ARG, "W0, W2 and W1 must not be NULL");
  if (d.momentum && !alpha && d.N > 0)
    return fail(TTT_ERR_INVALID_ARG, "momentum needs alpha [B,H,C]");
  if (d.N > 0) {
    if (!q || !k || !v || !eta || !out)
      return fail(TTT_ERR_INVALID_ARG, "q, k, v, eta and out must not be NULL");
    if (!al16(q) || !al16(k) || !al16(v) || !al16(out) || !al16(W0) || !al16(W2) || !al16(W1))
      return fail(TTT_ERR_INVALID_ARG, "q, k, v, out and the weights must be 16-byte aligned");
  }
  RecBufs b;
  const size_t need = plan_recurrent(d, nullptr, b);
  TTT_TRY(check_ws(workspace, workspace_bytes, need));
  t_guards.clear();
  plan_recurrent(d, workspace, b);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int ot = d.dtype == TTT_DTYPE_BF16 ? DT_BF16 : DT_F32;
  TTT_TRY(checks_begin(s));
  // every operand copy starts from the initial weights (a matrix outside the update mask is
  // never rewritten): the set-up kernels write all three copies
  TTT_OP("rec_init", rec_init(ot, W0, W2, W1, (int)BH, d.H, d.h, d.m, b.W_all, b.W1t[0],
                              d.momentum ? M_io : nullptr, b.M_all, d.momentum, s, b.W1t[1],
                              b.W1t[2]));
  TTT_OP("prep_weights", prep_wk_blocked(ot, W0, W2, b.Wk[0], (int)BH, d.H, d.h, d.m, 0, s,
                                         b.Wk[1], b.Wk[2]));
  if (d.renorm) TTT_OP("col_norms", col_norms(W0, W2, W1, d.H, d.h, d.m, b.tnorm, s));
  const long long N = d.N, L = d.chunk;
  // The apply of chunk c - 1 (update -> apply order; of chunk c in apply -> update order)
  // and the update of chunk c read the same operand copy and write disjoint buffers, so the
  // applies run on a second stream, each released by the gate event of update c (at its
  // Newton-Schulz kernel, which leaves most SMs idle, or at its start); each update waits
  // for the apply that last read the operand copy it is about to overwrite: with three
  // copies, the apply enqueued two iterations earlier.
  SideStream* side = side_stream();
  const bool fork = side != nullptr && N > L;
  const bool ua = d.order == TTT_ORDER_UPDATE_APPLY;
  cudaStream_t sa = fork ? side->s : s;
  auto chunks = [&]() -> ttt_status {
    int c = 0;
    for (long long t0 = 0; t0 < N; t0 += L, ++c) {
      const long long Lc = (t0 + L <= N) ? L : N - t0;
      const int bin = c % 3, bout = (c + 1) % 3;
      // update c writes copy bout; the apply enqueued two iterations earlier read it
      if (fork && (ua ? c >= 3 : c >= 2))
        TTT_CUDA(cudaStreamWaitEvent(s, side->applied[(c - 2) % 3], 0));
      TTT_TRY(rec_update(d, k, v, eta, alpha, c, t0, Lc, b, bin, bout, fork ? side : nullptr,
                         s));
      // the apply that reads copy bin (the weights after update c - 1): of chunk c - 1 in
      // update -> apply order, of chunk c in apply -> update order
      if (ua && c == 0) continue;
      const long long ta = ua ? t0 - L : t0, La = ua ? L : Lc;
      if (fork) TTT_CUDA(cudaStreamWaitEvent(sa, side->gate, 0));
      TTT_TRY(rec_apply(d, q, out, ta, La, b, bin, sa));
      if (fork) TTT_CUDA(cudaEventRecord(side->applied[c % 3], sa));
    }
    if (ua && c > 0) {   // the last chunk's apply, after the last update
      const long long ta = (long long)(c - 1) * L;
      if (fork) {
        TTT_CUDA(cudaEventRecord(side->gate, s));
        TTT_CUDA(cudaStreamWaitEvent(sa, side->gate, 0));
      }
      TTT_TRY(rec_apply(d, q, out, ta, N - ta, b, c % 3, sa));
    }
    return TTT_OK;
  };
  const ttt_status st = chunks();
  // join on every path: the caller's stream is ordered after every apply
  if (fork) {
    const cudaError_t e1 = cudaEventRecord(side->joined, sa);
    const cudaError_t e2 = e1 == cudaSuccess ? cudaStreamWaitEvent(s, side->joined, 0) : e1;
    if (st == TTT_OK && e2 != cudaSuccess)
      return fail(TTT_ERR_CUDA, "joining the apply stream: %s", cudaGetErrorString(e2));
  }
  TTT_TRY(st);
  if (W0_out || W2_out || W1_out || (d.momentum && M_io))
    TTT_OP("rec_finish", rec_finish(b.W_all, (int)BH, d.H, d.h, d.m, W0_out, W2_out, W1_out,
                                    b.M_all, d.momentum ? M_io : nullptr, s));
  const long long hm = (long long)d.h * d.m;
  return checks_end(s, {{out, BH * N * d.h, ot}, {W0_out, BH * hm, DT_F32},
                        {W2_out, BH * hm, DT_F32}, {W1_out, BH * hm, DT_F32},
                        {d.momentum ? M_io : nullptr, BH * 3 * hm, DT_F32}});
}

}  // extern "C"

// ------------------------------------------------------------------ built-in scratch
// Scratch of ttt_la_parallel_fwd_noalloc: one array per device, part of the library's
// device image, so the entry point never allocates. Its address is looked up once per
// device with that device current.
namespace ttt {
namespace {
static __device__ __align__(256) unsigned char g_static_scratch[TTT_STATIC_SCRATCH_BYTES];

ttt_status static_scratch(void** out) {
  static std::mutex mu;
  static void* addr[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(TTT_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 128) return fail(TTT_ERR_UNSUPPORTED, "device index %d >= 128", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p)
      return fail(TTT_ERR_CUDA, "cudaGetSymbolAddress(built-in scratch): %s",
                  cudaGetErrorString(e));
    addr[dev] = p;
  }
  *out = addr[dev];
  return TTT_OK;
}
}  // namespace
}  // namespace ttt

extern "C" {

ttt_status ttt_la_parallel_fwd_noalloc(const ttt_desc* desc, const void* q, const void* k,
                                       const void* v, const float* eta, const float* W0,
                                       const float* W2, const float* W1, void* out,
                                       float* S_final, ttt_stream_t stream) {
  TTT_TRY(check_desc(desc, TTT_PATH_PARALLEL));
  ParBufs b;
  const size_t need = plan_parallel(*desc, nullptr, b, sequential_schedule(*desc));
  if (need > TTT_STATIC_SCRATCH_BYTES)
    return fail(TTT_ERR_WORKSPACE,
                "problem needs %zu bytes of scratch; the built-in scratch holds %llu bytes "
                "(use ttt_la_parallel_fwd with a caller workspace)",
                need, (unsigned long long)TTT_STATIC_SCRATCH_BYTES);
  void* scratch = nullptr;
  TTT_TRY(static_scratch(&scratch));
  return ttt_la_parallel_fwd(desc, q, k, v, eta, W0, W2, W1, out, S_final, scratch,
                             (size_t)TTT_STATIC_SCRATCH_BYTES, stream);
}

size_t ttt_lm_target_workspace_bytes(int32_t N, int32_t d) {
  if (N < 0 || d < 1) return 0;
  Carve cv(nullptr);
  cv.take(2 * (size_t)N * d);
  return cv.off;
}

ttt_status ttt_lm_target(int32_t N, int32_t d, const void* X0, const float* conv_w,
                         const void* W_target, void* vbar, void* workspace,
                         size_t workspace_bytes, ttt_stream_t stream) {
  if (N < 0 || d < 1) return fail(TTT_ERR_INVALID_ARG, "N must be >= 0 and d >= 1");
  if (d % 8 != 0) return fail(TTT_ERR_UNSUPPORTED, "d must be a multiple of 8");
  if (N > (1 << 22)) return fail(TTT_ERR_UNSUPPORTED, "N must be <= 4194304");
  if (N == 0) return TTT_OK;
  if (!X0 || !conv_w || !W_target || !vbar)
    return fail(TTT_ERR_INVALID_ARG, "X0, conv_w, W_target and vbar must not be NULL");
  if (!al16(X0) || !al16(W_target) || !al16(vbar))
    return fail(TTT_ERR_INVALID_ARG, "X0, W_target and vbar must be 16-byte aligned");
  const size_t need = ttt_lm_target_workspace_bytes(N, d);
  TTT_TRY(check_ws(workspace, workspace_bytes, need));
  t_guards.clear();
  Carve cv(workspace);
  void* Xc = cv.take(2 * (size_t)N * d);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return with_checks(s, {{vbar, (long long)N * d, DT_BF16}}, [&]() -> ttt_status {
    TTT_OP("conv4_causal", conv4_causal(X0, conv_w, Xc, N, d, s));
    GemmProblem p;
    p.M = N; p.N = d; p.K = d;
    p.A = {Xc, DT_BF16, false, d, 0, 0};
    p.B = {W_target, DT_BF16, true, d, 0, 0};
    p.C = {vbar, DT_BF16, d, 0, 0};
    return run_gemm("gemm_lm_target", p, s);
  });
}

ttt_status ttt_last_device_status(ttt_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(TTT_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  unsigned w = 0;
  e = cudaMemcpyFromSymbol(&w, g_dev_err_word, sizeof(w));
  if (e != cudaSuccess) return fail(TTT_ERR_CUDA, "read error word: %s", cudaGetErrorString(e));
  if (w) {
    const unsigned z = 0;
    cudaMemcpyToSymbol(g_dev_err_word, &z, sizeof(z));
    if (w & DEVERR_TIMEOUT) return fail(TTT_ERR_TIMEOUT, "a bounded device wait ran out");
    if (w & DEVERR_BOUNDS)
      return fail(TTT_ERR_DEVICE, "a workspace guard was overwritten: a write went outside its "
                  "region (word 0x%x)", w);
    if (w & DEVERR_NONFINITE)
      return fail(TTT_ERR_DEVICE, "an output holds NaN or Inf (word 0x%x)", w);
    return fail(TTT_ERR_DEVICE, "device-side check failed (word 0x%x)", w);
  }
  return TTT_OK;
}

ttt_status ttt_set_debug_checks(int32_t flags) {
  if (flags & ~(TTT_CHECK_GUARDS | TTT_CHECK_FINITE))
    return fail(TTT_ERR_INVALID_ARG, "unknown debug check flags 0x%x", (unsigned)flags);
  g_checks.store(flags);
  return TTT_OK;
}

int32_t ttt_get_debug_checks(void) { return g_checks.load(); }

ttt_status ttt_debug_check_workspace(const ttt_desc* desc, int32_t path, void* workspace,
                                     size_t workspace_bytes, ttt_stream_t stream) {
  if (!(g_checks.load() & TTT_CHECK_GUARDS))
    return fail(TTT_ERR_INVALID_ARG, "workspace guards are off (TTT_CHECK_GUARDS)");
  TTT_TRY(check_desc(desc, path));
  const size_t need = ttt_workspace_bytes(desc, path);
  TTT_TRY(check_ws(workspace, workspace_bytes, need));
  t_guards.clear();
  switch (path) {
    case TTT_PATH_PARALLEL: {
      ParBufs b;
      plan_parallel(*desc, workspace, b, sequential_schedule(*desc));
      break;
    }
    case TTT_PATH_LINEAR: { LinBufs b; plan_linear(*desc, workspace, b); break; }
    case TTT_PATH_PARALLEL_MOMENTUM: { MomBufs b; plan_momentum(*desc, workspace, b); break; }
    case TTT_PATH_PARALLEL_BWD: { BwdBufs b; plan_backward(*desc, workspace, b); break; }
    default: { RecBufs b; plan_recurrent(*desc, workspace, b); break; }
  }
  return run_guards(true, reinterpret_cast<cudaStream_t>(stream));
}

ttt_status ttt_debug_wait_timeout(int64_t timeout_ns, ttt_stream_t stream) {
  if (timeout_ns < 100000 || timeout_ns > 10000000000LL)
    return fail(TTT_ERR_INVALID_ARG, "timeout_ns must be in [1e5, 1e10]");
  unsigned* w = device_error_word();
  if (!w) return fail(TTT_ERR_CUDA, "no device error word");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  TTT_OP("wait_timeout_probe", wait_timeout_probe(w, (unsigned long long)timeout_ns, s));
  return TTT_OK;
}

ttt_status ttt_trace_enable(int32_t capacity) {
  if (capacity < 1 || capacity > (1 << 20))
    return fail(TTT_ERR_INVALID_ARG, "trace capacity must be in 1..2^20");
  ttt_trace_disable();
  std::lock_guard<std::mutex> lk(g_trace.mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(TTT_ERR_CUDA, "cudaGetDevice failed");
  g_trace.ev.assign(2 * (size_t)capacity, nullptr);
  for (auto& e : g_trace.ev)
    if (cudaEventCreate(&e) != cudaSuccess) return fail(TTT_ERR_CUDA, "cudaEventCreate failed");
  g_trace.names.assign(capacity, "");
  g_trace.cap = capacity;
  g_trace.n = 0;
  g_trace.dev = dev;
  g_trace.on = true;
  return TTT_OK;
}

ttt_status ttt_trace_disable(void) {
  std::lock_guard<std::mutex> lk(g_trace.mu);
  g_trace.on = false;
  for (auto& e : g_trace.ev)
    if (e) cudaEventDestroy(e);
  g_trace.ev.clear();
  g_trace.names.clear();
  g_trace.n = g_trace.cap = 0;
  return TTT_OK;
}

int32_t ttt_trace_count(void) { return g_trace.n; }

ttt_status ttt_trace_get(int32_t index, const char** kernel_name, float* milliseconds) {
  std::lock_guard<std::mutex> lk(g_trace.mu);
  if (index < 0 || index >= g_trace.n) return fail(TTT_ERR_INVALID_ARG, "trace index out of range");
  cudaEvent_t a = g_trace.ev[2 * (size_t)index], b = g_trace.ev[2 * (size_t)index + 1];
  if (cudaEventSynchronize(b) != cudaSuccess) return fail(TTT_ERR_CUDA, "cudaEventSynchronize failed");
  float ms = 0.0f;
  if (cudaEventElapsedTime(&ms, a, b) != cudaSuccess)
    return fail(TTT_ERR_CUDA, "cudaEventElapsedTime failed");
  if (kernel_name) *kernel_name = g_trace.names[index];
  if (milliseconds) *milliseconds = ms;
  return TTT_OK;
}

const char* ttt_status_str(ttt_status status) {
  switch (status) {
    case TTT_OK: return "TTT_OK";
    case TTT_ERR_INVALID_ARG: return "TTT_ERR_INVALID_ARG";
    case TTT_ERR_UNSUPPORTED: return "TTT_ERR_UNSUPPORTED";
    case TTT_ERR_WORKSPACE: return "TTT_ERR_WORKSPACE";
    case TTT_ERR_CUDA: return "TTT_ERR_CUDA";
    case TTT_ERR_TIMEOUT: return "TTT_ERR_TIMEOUT";
    case TTT_ERR_DEVICE: return "TTT_ERR_DEVICE";
  }
  return "TTT_ERR_UNKNOWN";
}

const char* ttt_last_error_message(void) { return g_msg; }

int32_t ttt_version(void) { return 100; }

}  // extern "C"
