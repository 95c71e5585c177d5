// Host side of the C ABI declared in include/mmf.h: argument validation,
// workspace carving and the launch sequence of each entry point.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "kernels.cuh"

using namespace mmf;

// ------------------------------------------------------------------ errors

namespace {

thread_local std::string g_last_error;

mmf_status fail(mmf_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

mmf_status cuda_fail(cudaError_t e, const char* where) {
  return fail(MMF_ERR_CUDA, "%s: CUDA error %d (%s)", where, (int)e, cudaGetErrorString(e));
}

#define MMF_CUDA(call, where)                      \
  do {                                             \
    cudaError_t e_ = (call);                       \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline size_t elem_bytes(mmf_dtype dt) { return dt == MMF_BF16 ? 2 : 4; }
inline bool dtype_ok(mmf_dtype dt) { return dt == MMF_F32 || dt == MMF_BF16; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Bump allocator over the caller's workspace (256-byte granules).
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T> T* take(size_t count) {
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += round_up(sizeof(T) * count, 256);
    return p;
  }
};

// Per-device status word written by kernels that give up a bounded wait.
constexpr int kMaxDevices = 64;
int* g_dev_status[kMaxDevices] = {};
std::mutex g_dev_status_mu;

mmf_status device_status_ptr(int** out) {
  int dev = 0;
  MMF_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MMF_ERR_INVALID_ARG, "device %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_status_mu);
  if (g_dev_status[dev] == nullptr) {
    int* p = nullptr;
    MMF_CUDA(cudaMalloc(&p, sizeof(int)), "cudaMalloc(status word)");
    MMF_CUDA(cudaMemset(p, 0, sizeof(int)), "cudaMemset(status word)");
    g_dev_status[dev] = p;
  }
  *out = g_dev_status[dev];
  return MMF_OK;
}

// ------------------------------------------------------------------ launch timing
// Every launch goes through timed(): when the profiler is on, two CUDA events
// bracket it on its stream; mmf_prof_collect folds finished pairs into totals.
struct ProfPair {
  int kind;
  cudaEvent_t a, b;
};
struct ProfKind {
  std::string name;
  long long launches = 0;
  double ms = 0.0;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfPair> g_prof_pending;
std::vector<cudaEvent_t> g_prof_free;
std::vector<ProfKind> g_prof_kinds;

cudaEvent_t prof_event() {
  if (!g_prof_free.empty()) {
    cudaEvent_t e = g_prof_free.back();
    g_prof_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

int prof_kind(const char* name) {
  for (size_t i = 0; i < g_prof_kinds.size(); ++i)
    if (g_prof_kinds[i].name == name) return (int)i;
  g_prof_kinds.push_back(ProfKind{name});
  return (int)g_prof_kinds.size() - 1;
}

template <class F>
cudaError_t timed(const char* name, cudaStream_t s, F&& launch) {
  if (!g_prof_on) return launch();
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaEvent_t a = prof_event(), b = prof_event();
  if (a) cudaEventRecord(a, s);
  cudaError_t e = launch();
  if (b) cudaEventRecord(b, s);
  if (a && b) g_prof_pending.push_back(ProfPair{prof_kind(name), a, b});
  return e;
}

// Contraction dispatch: the single-SM tcgen05 kernel from 128 tokens, the
// mma.sync kernel for decode-sized token counts and for shapes the tcgen05
// kernels do not take. The SM-pair tcgen05 kernel (M >= 256) is selected only
// on request: it is correct but measured slower than the single-SM kernel on
// the 370M shapes. MMF_GEMM_PATH=mma|tc|tc1|tc2|auto (default auto; tc and tc1
// both mean the single-SM kernel) pins one implementation; all compute the
// same exact integer accumulators.
constexpr int kTcMinTokens = 128;

int gemm_path_pref() {
  const char* e = getenv("MMF_GEMM_PATH");
  if (e == nullptr) return 0;
  if (strcmp(e, "mma") == 0) return 1;
  if (strcmp(e, "tc") == 0) return 2;
  if (strcmp(e, "tc1") == 0) return 3;
  if (strcmp(e, "tc2") == 0) return 4;
  return 0;
}

// The prefill token mixer as one kernel (contraction + MLGRU in the epilogue)
// only with MMF_FUSED_MLGRU=1: it saves the pre-activation round trip through
// HBM, but its epilogue (gates and a warp-shuffle scan per channel) takes
// about twice as long as the contraction's main loop, and on one B200 it
// measured 3.9 ms per 370M step against 3.0 ms for contraction + scan.
bool fused_mlgru_enabled() {
  const char* e = getenv("MMF_FUSED_MLGRU");
  return e != nullptr && strcmp(e, "1") == 0;
}

bool gemm_uses_tc(const TGemmArgs& a, Epi epi) {
  const int pref = gemm_path_pref();
  return tgemm_tc_supported(a, epi) && (pref >= 2 || (pref == 0 && a.M >= kTcMinTokens));
}

// Whether the decode contraction quantises its own token rows (both ways give
// the same codes). Every CTA then repeats the row work, which on one B200 beat
// the standalone quantiser plus one kernel boundary only for single-token
// calls (1.3B decode at 4 tokens: 0.69 ms per step fused, 0.59 ms split).
// MMF_DECODE_FUSED_QUANT=1 fuses whenever the shapes allow, =0 never.
bool decode_fused_quant_wanted(int M) {
  const char* e = getenv("MMF_DECODE_FUSED_QUANT");
  if (e != nullptr && strcmp(e, "1") == 0) return true;
  if (e != nullptr && strcmp(e, "0") == 0) return false;
  return M == 1;
}

// `what` names the projection for the launch-timing totals ("fcg", "o", ...).
cudaError_t run_gemm(const TGemmArgs& a, Epi epi, mmf_dtype dt, cudaStream_t s, const char* what = "") {
  const int pref = gemm_path_pref();
  const bool tc2_ok = tgemm_tc2_supported(a, epi);
  bool use_tc = gemm_uses_tc(a, epi);
  const bool use_tc2 = use_tc && tc2_ok && pref == 4;
  char name[48];
  snprintf(name, sizeof(name), "%s%s%s", use_tc2 ? "tgemm_tc2" : (use_tc ? "tgemm_tc" : "tgemm_mma"),
           what[0] ? ":" : "", what);
  if (use_tc) {
    int* st = nullptr;
    if (device_status_ptr(&st) != MMF_OK) return cudaErrorUnknown;
    if (use_tc2) return timed(name, s, [&] { return launch_tgemm_tc2(a, epi, dt, st, s); });
    return timed(name, s, [&] { return launch_tgemm_tc(a, epi, dt, st, s); });
  }
  return timed(name, s, [&] { return launch_tgemm_mma(a, epi, dt, s); });
}

// Device status word for kernels with bounded waits, or null when it cannot be had.
int* status_word() {
  int* st = nullptr;
  return device_status_ptr(&st) == MMF_OK ? st : nullptr;
}

// Quantised activations of M tokens of length K.
struct QAct {
  int8_t* q;
  float* s;
  int32_t* qsum;
};

// RMSNorm + int8 quantisation of x (a.M tokens of length a.K, RMSNorm gain
// `gain`), then the contraction `a` (whose q/s/qsum point at qa). Single-token
// calls on the mma.sync kernel quantise inside the contraction (one launch);
// the codes also land in qa when `want_codes`. Otherwise the quantiser fills qa
// and the contraction reads it.
mmf_status quant_gemm(const void* x, const float* gain, float eps, const QAct& qa, TGemmArgs a, Epi epi,
                      mmf_dtype dt, cudaStream_t s, const char* what, bool want_codes, void* fill = nullptr,
                      size_t fill_bytes = 0) {
  if (!gemm_uses_tc(a, epi) && decode_fused_quant_wanted(a.M) &&
      tgemm_mma_fused_quant_supported(a.M, a.K, elem_bytes(dt))) {
    if (fill_bytes) MMF_CUDA(cudaMemsetAsync(fill, 0xff, fill_bytes, s), "scratch fill");
    a.x = x;
    a.gain = gain;
    a.eps = eps;
    a.q_out = want_codes ? qa.q : nullptr;
    a.s_out = want_codes ? qa.s : nullptr;
    a.qsum_out = want_codes ? qa.qsum : nullptr;
    MMF_CUDA(run_gemm(a, epi, dt, s, what), "fused quant + contraction");
    return MMF_OK;
  }
  MMF_CUDA(timed("rmsnorm_quant", s,
                 [&] {
                   return launch_rmsnorm_quant(x, dt, a.M, a.K, gain, eps, qa.q, qa.s, qa.qsum, status_word(), s,
                                               fill, fill_bytes);
                 }),
           "rmsnorm_quant");
  MMF_CUDA(run_gemm(a, epi, dt, s, what), "contraction");
  return MMF_OK;
}

// Blocks keep one-byte copies of their codes for the prefill contraction
// (4x the packed weight memory) unless MMF_PREFILL_UNPACKED=0.
bool prefill_unpacked_enabled() {
  const char* e = getenv("MMF_PREFILL_UNPACKED");
  return e == nullptr || strcmp(e, "0") != 0;
}

mmf_status check_tlinear(const mmf_tlinear* l, const char* name) {
  if (l == nullptr) return fail(MMF_ERR_INVALID_ARG, "%s: null layer", name);
  if (l->packed == nullptr || l->gamma == nullptr) return fail(MMF_ERR_INVALID_ARG, "%s: null packed/gamma", name);
  if (l->N < 1 || l->K < 1) return fail(MMF_ERR_INVALID_ARG, "%s: N=%d K=%d must be >= 1", name, l->N, l->K);
  if (l->K % 16 != 0) return fail(MMF_ERR_UNSUPPORTED_SHAPE, "%s: K=%d is not a multiple of 16", name, l->K);
  if (!aligned16(l->packed)) return fail(MMF_ERR_MISALIGNED, "%s: packed not 16-byte aligned", name);
  if ((l->gain && !aligned16(l->gain)) || (l->bias && !aligned16(l->bias)) || (l->codes && !aligned16(l->codes)))
    return fail(MMF_ERR_MISALIGNED, "%s: gain/bias/codes not 16-byte aligned", name);
  return MMF_OK;
}

TGemmArgs gemm_args(const mmf_tlinear* const* segs, int nseg, const int8_t* q, const float* s,
                    const int32_t* qsum, int M, void* out, int ldo, const void* residual, float* h) {
  TGemmArgs a{};
  for (int i = 0; i < 3; ++i) {
    const mmf_tlinear* l = segs[i < nseg ? i : 0];
    a.w[i] = l->packed;
    a.wu[i] = l->codes;
    a.gamma[i] = l->gamma;
    a.bias[i] = l->bias;
  }
  a.nseg = nseg;
  a.N = segs[0]->N;
  a.K = segs[0]->K;
  a.q = q;
  a.s = s;
  a.qsum = qsum;
  a.M = M;
  a.out = out;
  a.ldo = ldo;
  a.residual = residual;
  a.h = h;
  return a;
}


QAct carve_qact(Carver& c, int M, int K) {
  QAct a;
  a.q = c.take<int8_t>((size_t)M * K);
  a.s = c.take<float>(M);
  a.qsum = c.take<int32_t>(M);
  return a;
}

}  // namespace

void mmf::set_last_error(const char* msg) { g_last_error = msg; }

// ------------------------------------------------------------------ handles

// wu: one-byte codes of the seven matrices (f, c, g, o, gate, up, down) for
// the prefill contraction: the caller's mmf_tlinear.codes, or copies made at
// creation (owned[i]); all null when disabled.
struct mmf_block {
  mmf_block_weights w;
  int d, I;
  const uint8_t* wu[7];
  uint8_t* owned[7];
};

// bar: 256 bytes holding the counter and generation words of the one-launch
// decode step's grid barrier, zero between launches; calls sharing a state are stream-ordered
// anyway (h is updated in place), so one pair serves every layer.
struct mmf_state {
  float* h;
  unsigned* bar;
  int L, B, d;
};

// ------------------------------------------------------------------ misc

extern "C" const char* mmf_version(void) { return "mmf 0.1.0 sm_100a"; }

extern "C" const char* mmf_last_error(void) { return g_last_error.c_str(); }

extern "C" mmf_status mmf_check(void* stream) {
  MMF_CUDA(cudaStreamSynchronize(as_stream(stream)), "mmf_check: cudaStreamSynchronize");
  MMF_CUDA(cudaGetLastError(), "mmf_check: pending error");
  int* st = nullptr;
  mmf_status r = device_status_ptr(&st);
  if (r != MMF_OK) return r;
  int v = 0;
  MMF_CUDA(cudaMemcpy(&v, st, sizeof(int), cudaMemcpyDeviceToHost), "mmf_check: read status");
  if (v != 0) {
    MMF_CUDA(cudaMemset(st, 0, sizeof(int)), "mmf_check: clear status");
    return fail(MMF_ERR_TIMEOUT, "a device-side bounded wait gave up (code %d)", v);
  }
  return MMF_OK;
}

// ------------------------------------------------------------------ weights

extern "C" size_t mmf_quantize_weights_ws_size(int32_t N, int32_t K) {
  (void)N;
  (void)K;
  return quantize_weights_ws_bytes();
}

extern "C" mmf_status mmf_quantize_weights(const float* W, int32_t N, int32_t K, uint32_t* packed, float* gamma,
                                           void* ws, size_t ws_bytes, void* stream) {
  if (!W || !packed || !gamma || !ws) return fail(MMF_ERR_INVALID_ARG, "mmf_quantize_weights: null pointer");
  if (N < 1 || K < 1) return fail(MMF_ERR_INVALID_ARG, "mmf_quantize_weights: N=%d K=%d", N, K);
  if (K % 16 != 0) return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_quantize_weights: K=%d %% 16 != 0", K);
  if (!aligned16(W) || !aligned16(packed) || !aligned16(ws))
    return fail(MMF_ERR_MISALIGNED, "mmf_quantize_weights: pointer not 16-byte aligned");
  if (ws_bytes < mmf_quantize_weights_ws_size(N, K))
    return fail(MMF_ERR_WORKSPACE, "mmf_quantize_weights: ws_bytes=%zu < %zu", ws_bytes,
                mmf_quantize_weights_ws_size(N, K));
  MMF_CUDA(timed("quantize_weights", as_stream(stream),
                 [&] { return launch_quantize_weights(W, N, K, packed, gamma, ws, as_stream(stream)); }),
           "mmf_quantize_weights");
  return MMF_OK;
}

// ------------------------------------------------------------------ BitLinear

extern "C" size_t mmf_bitlinear_ws_size(int32_t M, int32_t K) {
  if (M < 0 || K < 0) return 0;
  Carver c(nullptr);
  carve_qact(c, M, K);
  return c.off + 256;
}

extern "C" mmf_status mmf_unpack_codes(const uint32_t* packed, int32_t N, int32_t K, uint8_t* codes, void* stream) {
  if (!packed || !codes) return fail(MMF_ERR_INVALID_ARG, "mmf_unpack_codes: null pointer");
  if (N < 1 || K < 1) return fail(MMF_ERR_INVALID_ARG, "mmf_unpack_codes: N=%d K=%d", N, K);
  if (K % 16 != 0) return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_unpack_codes: K=%d %% 16 != 0", K);
  if (!aligned16(packed) || !aligned16(codes)) return fail(MMF_ERR_MISALIGNED, "mmf_unpack_codes");
  MMF_CUDA(launch_unpack_codes(packed, N, K, codes, as_stream(stream)), "mmf_unpack_codes");
  return MMF_OK;
}

extern "C" mmf_status mmf_bitlinear(const mmf_tlinear* lin, const void* x, mmf_dtype dtype, int32_t M, void* y,
                                    float eps, void* ws, size_t ws_bytes, void* stream,
                                    const mmf_bitlinear_debug* dbg) {
  mmf_status st = check_tlinear(lin, "mmf_bitlinear");
  if (st != MMF_OK) return st;
  if (!dtype_ok(dtype)) return fail(MMF_ERR_INVALID_ARG, "mmf_bitlinear: bad dtype %d", (int)dtype);
  if (M < 0) return fail(MMF_ERR_INVALID_ARG, "mmf_bitlinear: M=%d", M);
  if (!(eps > 0.0f)) return fail(MMF_ERR_INVALID_ARG, "mmf_bitlinear: eps must be > 0");
  if (M == 0) return MMF_OK;
  if (!x || !y || !ws) return fail(MMF_ERR_INVALID_ARG, "mmf_bitlinear: null x/y/ws");
  if (!aligned16(x) || !aligned16(y) || !aligned16(ws)) return fail(MMF_ERR_MISALIGNED, "mmf_bitlinear: x/y/ws");
  if (dbg && ((dbg->q && !aligned16(dbg->q)) || (dbg->acc && !aligned16(dbg->acc))))
    return fail(MMF_ERR_MISALIGNED, "mmf_bitlinear: debug buffers");
  if (ws_bytes < mmf_bitlinear_ws_size(M, lin->K))
    return fail(MMF_ERR_WORKSPACE, "mmf_bitlinear: ws_bytes=%zu < %zu", ws_bytes, mmf_bitlinear_ws_size(M, lin->K));
  cudaStream_t s = as_stream(stream);
  const mmf_tlinear* segs[1] = {lin};
  Carver c(ws);
  QAct qa = carve_qact(c, M, lin->K);
  TGemmArgs a = gemm_args(segs, 1, qa.q, qa.s, qa.qsum, M, y, lin->N, nullptr, nullptr);
  mmf_status r = quant_gemm(x, lin->gain, eps, qa, a, Epi::kStore, dtype, s, "", dbg != nullptr);
  if (r != MMF_OK) return r;
  if (dbg) {
    if (dbg->q) MMF_CUDA(cudaMemcpyAsync(dbg->q, qa.q, (size_t)M * lin->K, cudaMemcpyDeviceToDevice, s), "dbg q");
    if (dbg->scale)
      MMF_CUDA(cudaMemcpyAsync(dbg->scale, qa.s, sizeof(float) * M, cudaMemcpyDeviceToDevice, s), "dbg scale");
    if (dbg->acc) {
      TGemmArgs d = gemm_args(segs, 1, qa.q, qa.s, qa.qsum, M, dbg->acc, lin->N, nullptr, nullptr);
      MMF_CUDA(run_gemm(d, Epi::kAcc, dtype, s), "tgemm acc");
    }
  }
  return MMF_OK;
}

// ------------------------------------------------------------------ MLGRU scan

extern "C" size_t mmf_mlgru_scan_ws_size(int32_t B, int32_t T, int32_t d) {
  if (B < 0 || T < 0 || d < 0) return 0;
  return mlgru_scan_ws_bytes(B, T, d);
}

extern "C" mmf_status mmf_mlgru_scan(const void* pre, mmf_dtype dtype, int32_t B, int32_t T, int32_t d, float* h,
                                     void* o, void* ws, size_t ws_bytes, void* stream) {
  if (!dtype_ok(dtype)) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan: bad dtype");
  if (B < 0 || T < 0 || d < 1) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan: B=%d T=%d d=%d", B, T, d);
  if (d % 8 != 0) return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_mlgru_scan: d=%d %% 8 != 0", d);
  if (B == 0 || T == 0) return MMF_OK;
  if (!pre || !h || !o || !ws) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan: null pointer");
  if (!aligned16(pre) || !aligned16(h) || !aligned16(o) || !aligned16(ws))
    return fail(MMF_ERR_MISALIGNED, "mmf_mlgru_scan");
  if (ws_bytes < mlgru_scan_ws_bytes(B, T, d))
    return fail(MMF_ERR_WORKSPACE, "mmf_mlgru_scan: ws_bytes=%zu < %zu", ws_bytes, mlgru_scan_ws_bytes(B, T, d));
  cudaStream_t s = as_stream(stream);
  int* status = nullptr;
  mmf_status r = device_status_ptr(&status);
  if (r != MMF_OK) return r;
  MMF_CUDA(timed("mlgru_scan", s,
                 [&] {
                   cudaError_t e = reset_mlgru_scan_ws(ws, B, T, d, s);
                   return e != cudaSuccess ? e : launch_mlgru_scan(pre, dtype, B, T, d, h, o, ws, status, s);
                 }),
           "mlgru_scan");
  return MMF_OK;
}

// ------------------------------------------------------------------ GLU

namespace {

size_t glu_ws(int M, int d, int I, mmf_dtype dt) {
  Carver c(nullptr);
  carve_qact(c, M, std::max(d, I));
  c.take<char>((size_t)M * I * elem_bytes(dt));
  return c.off + 256;
}

mmf_status check_glu(const mmf_tlinear* gate, const mmf_tlinear* up, const mmf_tlinear* down, int d) {
  mmf_status st;
  if ((st = check_tlinear(gate, "gate")) != MMF_OK) return st;
  if ((st = check_tlinear(up, "up")) != MMF_OK) return st;
  if ((st = check_tlinear(down, "down")) != MMF_OK) return st;
  if (gate->K != d || up->K != d || up->N != gate->N || down->K != gate->N || down->N != d)
    return fail(MMF_ERR_UNSUPPORTED_SHAPE, "glu: shapes gate %dx%d up %dx%d down %dx%d disagree", gate->N, gate->K,
                up->N, up->K, down->N, down->K);
  if (gate->gain != up->gain) return fail(MMF_ERR_UNSUPPORTED_SHAPE, "glu: gate and up must share one gain");
  return MMF_OK;
}

// p = SiLU(gate(x)) * up(x); y = down(p) + residual. x is quantised with the
// gate's RMSNorm gain (gate and up share it), p with the down projection's.
mmf_status run_glu(const mmf_tlinear* gate, const mmf_tlinear* up, const mmf_tlinear* down, const void* x,
                   const void* residual, void* y, int M, mmf_dtype dt, float eps, void* p, const QAct& qa,
                   cudaStream_t s, const uint8_t* const* wu = nullptr /* gate, up, down one-byte codes */) {
  const mmf_tlinear* gu[2] = {gate, up};
  TGemmArgs a = gemm_args(gu, 2, qa.q, qa.s, qa.qsum, M, p, gate->N, nullptr, nullptr);
  if (wu) {
    a.wu[0] = wu[0];
    a.wu[1] = wu[1];
  }   // otherwise the layers' own codes (if any), set by gemm_args
  mmf_status r = quant_gemm(x, gate->gain, eps, qa, a, Epi::kGlu, dt, s, "gate_up", false);
  if (r != MMF_OK) return r;
  const mmf_tlinear* dn[1] = {down};
  TGemmArgs b = gemm_args(dn, 1, qa.q, qa.s, qa.qsum, M, y, down->N, residual, nullptr);
  if (wu) b.wu[0] = wu[2];
  return quant_gemm(p, down->gain, eps, qa, b, Epi::kStore, dt, s, "down", false);
}

}  // namespace

extern "C" size_t mmf_glu_ws_size(int32_t M, int32_t d, int32_t I) {
  if (M < 0 || d < 0 || I < 0) return 0;
  return glu_ws(M, d, I, MMF_F32);
}

extern "C" mmf_status mmf_glu(const mmf_tlinear* gate, const mmf_tlinear* up, const mmf_tlinear* down,
                              const void* x, const void* residual, void* y, int32_t M, mmf_dtype dtype, float eps,
                              void* ws, size_t ws_bytes, void* stream) {
  if (!dtype_ok(dtype)) return fail(MMF_ERR_INVALID_ARG, "mmf_glu: bad dtype");
  if (M < 0) return fail(MMF_ERR_INVALID_ARG, "mmf_glu: M=%d", M);
  if (!(eps > 0.0f)) return fail(MMF_ERR_INVALID_ARG, "mmf_glu: eps must be > 0");
  if (!gate) return fail(MMF_ERR_INVALID_ARG, "mmf_glu: null gate");
  const int d = gate->K;
  mmf_status st = check_glu(gate, up, down, d);
  if (st != MMF_OK) return st;
  if (M == 0) return MMF_OK;
  if (!x || !y || !ws) return fail(MMF_ERR_INVALID_ARG, "mmf_glu: null x/y/ws");
  if (!aligned16(x) || !aligned16(y) || !aligned16(ws) || (residual && !aligned16(residual)))
    return fail(MMF_ERR_MISALIGNED, "mmf_glu: pointer not 16-byte aligned");
  const int I = gate->N;
  if (ws_bytes < mmf_glu_ws_size(M, d, I))
    return fail(MMF_ERR_WORKSPACE, "mmf_glu: ws_bytes=%zu < %zu", ws_bytes, mmf_glu_ws_size(M, d, I));
  cudaStream_t s = as_stream(stream);
  Carver c(ws);
  QAct qa = carve_qact(c, M, std::max(d, I));
  void* p = c.take<char>((size_t)M * I * elem_bytes(dtype));
  return run_glu(gate, up, down, x, residual, y, M, dtype, eps, p, qa, s);
}

// ------------------------------------------------------------------ blocks and state

extern "C" mmf_status mmf_block_create(const mmf_block_weights* w, int32_t d, int32_t I, mmf_block** out) {
  if (!w || !out) return fail(MMF_ERR_INVALID_ARG, "mmf_block_create: null pointer");
  *out = nullptr;
  if (d < 16 || I < 16) return fail(MMF_ERR_INVALID_ARG, "mmf_block_create: d=%d I=%d", d, I);
  mmf_status st;
  const mmf_tlinear* sq[4] = {&w->f, &w->c, &w->g, &w->o};
  const char* names[4] = {"f", "c", "g", "o"};
  for (int i = 0; i < 4; ++i) {
    if ((st = check_tlinear(sq[i], names[i])) != MMF_OK) return st;
    if (sq[i]->N != d || sq[i]->K != d)
      return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_block_create: %s is %dx%d, want %dx%d", names[i], sq[i]->N,
                  sq[i]->K, d, d);
  }
  if (w->f.gain != w->c.gain || w->f.gain != w->g.gain)
    return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_block_create: f, c and g must share one gain");
  if ((st = check_glu(&w->gate, &w->up, &w->down, d)) != MMF_OK) return st;
  if (w->gate.N != I) return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_block_create: gate N=%d != I=%d", w->gate.N, I);
  mmf_block* b = new (std::nothrow) mmf_block;
  if (!b) return fail(MMF_ERR_NOMEM, "mmf_block_create: out of host memory");
  b->w = *w;
  b->d = d;
  b->I = I;
  const mmf_tlinear* all[7] = {&w->f, &w->c, &w->g, &w->o, &w->gate, &w->up, &w->down};
  for (int i = 0; i < 7; ++i) {
    b->wu[i] = all[i]->codes;
    b->owned[i] = nullptr;
  }
  if (prefill_unpacked_enabled()) {
    // copies for the matrices the caller gave no codes for; they only speed
    // prefill up, so without device memory for them the block keeps using the
    // packed codes
    bool have = true;
    for (int i = 0; i < 7 && have; ++i) {
      if (b->wu[i] != nullptr) continue;
      if (cudaMalloc(&b->owned[i], (size_t)all[i]->N * all[i]->K) != cudaSuccess) {
        b->owned[i] = nullptr;
        have = false;
      }
    }
    if (!have) {
      (void)cudaGetLastError();   // clear the allocation error
      for (int i = 0; i < 7; ++i) {
        cudaFree(b->owned[i]);
        b->owned[i] = nullptr;
      }
    }
    bool launched = false;
    for (int i = 0; i < 7 && have; ++i) {
      if (b->owned[i] == nullptr) continue;
      cudaError_t e = launch_unpack_codes(all[i]->packed, all[i]->N, all[i]->K, b->owned[i], 0);
      if (e != cudaSuccess) {
        mmf_block_destroy(b);
        return cuda_fail(e, "mmf_block_create: unpack codes");
      }
      b->wu[i] = b->owned[i];
      launched = true;
    }
    if (launched) {
      cudaError_t e = cudaStreamSynchronize(0);
      if (e != cudaSuccess) {
        mmf_block_destroy(b);
        return cuda_fail(e, "mmf_block_create: synchronise");
      }
    }
  }
  *out = b;
  return MMF_OK;
}

extern "C" void mmf_block_destroy(mmf_block* blk) {
  if (!blk) return;
  for (int i = 0; i < 7; ++i) cudaFree(blk->owned[i]);
  delete blk;
}

extern "C" mmf_status mmf_state_create(int32_t L, int32_t B, int32_t d, mmf_state** out) {
  if (!out) return fail(MMF_ERR_INVALID_ARG, "mmf_state_create: null out");
  *out = nullptr;
  if (L < 1 || B < 1 || d < 1) return fail(MMF_ERR_INVALID_ARG, "mmf_state_create: L=%d B=%d d=%d", L, B, d);
  mmf_state* st = new (std::nothrow) mmf_state;
  if (!st) return fail(MMF_ERR_NOMEM, "mmf_state_create: out of host memory");
  const size_t bytes = sizeof(float) * (size_t)L * B * d;
  cudaError_t e = cudaMalloc(&st->h, bytes);
  if (e != cudaSuccess) {
    delete st;
    return fail(MMF_ERR_NOMEM, "mmf_state_create: cudaMalloc(%zu): %s", bytes, cudaGetErrorString(e));
  }
  e = cudaMalloc(&st->bar, 256);
  if (e != cudaSuccess) {
    cudaFree(st->h);
    delete st;
    return fail(MMF_ERR_NOMEM, "mmf_state_create: cudaMalloc(256): %s", cudaGetErrorString(e));
  }
  e = cudaMemset(st->h, 0, bytes);
  if (e == cudaSuccess) e = cudaMemset(st->bar, 0, 256);
  if (e != cudaSuccess) {
    cudaFree(st->h);
    cudaFree(st->bar);
    delete st;
    return cuda_fail(e, "mmf_state_create: cudaMemset");
  }
  st->L = L;
  st->B = B;
  st->d = d;
  *out = st;
  return MMF_OK;
}

extern "C" void mmf_state_destroy(mmf_state* st) {
  if (!st) return;
  cudaFree(st->h);
  cudaFree(st->bar);
  delete st;
}

extern "C" mmf_status mmf_state_reset(mmf_state* st, void* stream) {
  if (!st) return fail(MMF_ERR_INVALID_ARG, "mmf_state_reset: null state");
  MMF_CUDA(cudaMemsetAsync(st->h, 0, sizeof(float) * (size_t)st->L * st->B * st->d, as_stream(stream)),
           "mmf_state_reset");
  MMF_CUDA(cudaMemsetAsync(st->bar, 0, 256, as_stream(stream)), "mmf_state_reset: barrier words");
  return MMF_OK;
}

extern "C" uint32_t* mmf_state_barrier(mmf_state* st) { return st ? st->bar : nullptr; }

extern "C" float* mmf_state_layer(mmf_state* st, int32_t layer) {
  if (!st || layer < 0 || layer >= st->L) return nullptr;
  return st->h + (size_t)layer * st->B * st->d;
}

extern "C" mmf_status mmf_state_get(const mmf_state* st, float* host_dst, void* stream) {
  if (!st || !host_dst) return fail(MMF_ERR_INVALID_ARG, "mmf_state_get: null pointer");
  cudaStream_t s = as_stream(stream);
  MMF_CUDA(cudaMemcpyAsync(host_dst, st->h, sizeof(float) * (size_t)st->L * st->B * st->d, cudaMemcpyDeviceToHost, s),
           "mmf_state_get");
  MMF_CUDA(cudaStreamSynchronize(s), "mmf_state_get: sync");
  return MMF_OK;
}

extern "C" mmf_status mmf_state_set(mmf_state* st, const float* host_src, void* stream) {
  if (!st || !host_src) return fail(MMF_ERR_INVALID_ARG, "mmf_state_set: null pointer");
  cudaStream_t s = as_stream(stream);
  MMF_CUDA(cudaMemcpyAsync(st->h, host_src, sizeof(float) * (size_t)st->L * st->B * st->d, cudaMemcpyHostToDevice, s),
           "mmf_state_set");
  MMF_CUDA(cudaStreamSynchronize(s), "mmf_state_set: sync");
  return MMF_OK;
}

namespace {

struct BlockWs {
  QAct qa;     // quantised activations, [M, max(d, I)]
  void* pre;   // [M, 3, d] pre-activations (prefill only)
  void* og;    // [M, d] o' = g * h
  void* y1;    // [M, d] after the token mixer
  void* p;     // [M, I] GLU product
  void* ping;  // [M, d] stack intermediates
  void* pong;
  void* scan;  // scan scratch
  size_t bytes;
};

BlockWs carve_block(void* base, int B, int T, int d, int I, mmf_dtype dt) {
  const int M = B * T;
  Carver c(base);
  BlockWs w;
  const size_t e = elem_bytes(dt);
  w.qa = carve_qact(c, M, std::max(d, I));
  w.pre = c.take<char>((size_t)M * 3 * d * e);
  w.og = c.take<char>((size_t)M * d * e);
  w.y1 = c.take<char>((size_t)M * d * e);
  w.p = c.take<char>((size_t)M * I * e);
  w.ping = c.take<char>((size_t)M * d * e);
  w.pong = c.take<char>((size_t)M * d * e);
  w.scan = c.take<char>(std::max(mlgru_scan_ws_bytes(B, T, d), tgemm_tc_mlgru_ws_bytes(B, T, d)));
  w.bytes = c.off + 256;
  return w;
}

// With MMF_DECODE_BLOCK_KERNEL=1 a decode step of up to 8 tokens runs as one
// launch per block (four stages, grid barriers between them) instead of four
// contractions; both compute the same values. Off by default: on one B200 a
// 2.7B-shaped block step took 41.5 us that way against 29.1 us for the
// separate kernels (each stage's row quantisation, contraction and epilogue
// stay serial, and a grid barrier costs about as much as a kernel boundary
// with programmatic dependent launch).
bool decode_block_enabled() {
  const char* e = getenv("MMF_DECODE_BLOCK_KERNEL");
  return e != nullptr && strcmp(e, "1") == 0;
}

DecodeStage decode_stage(const mmf_tlinear* const* segs, int nseg) {
  DecodeStage st{};
  for (int i = 0; i < 3; ++i) {
    const mmf_tlinear* l = segs[i < nseg ? i : 0];
    st.w[i] = l->packed;
    st.gamma[i] = l->gamma;
    st.bias[i] = l->bias;
  }
  st.gain = segs[0]->gain;
  st.nseg = nseg;
  st.N = segs[0]->N;
  st.K = segs[0]->K;
  return st;
}

mmf_status block_forward_impl(const mmf_block* blk, float* h, unsigned* bar, const void* x, void* y, int B, int T,
                              mmf_dtype dt, float eps, const BlockWs& w, cudaStream_t s) {
  const int M = B * T, d = blk->d;
  const mmf_block_weights& W = blk->w;
  const mmf_tlinear* fcg[3] = {&W.f, &W.c, &W.g};
  if (T == 1 && decode_block_enabled()) {
    const mmf_tlinear* o1[1] = {&W.o};
    const mmf_tlinear* gu[2] = {&W.gate, &W.up};
    const mmf_tlinear* dn[1] = {&W.down};
    DecodeBlockArgs a{};
    a.st[0] = decode_stage(fcg, 3);
    a.st[1] = decode_stage(o1, 1);
    a.st[2] = decode_stage(gu, 2);
    a.st[3] = decode_stage(dn, 1);
    a.x = x;
    a.og = w.og;
    a.y1 = w.y1;
    a.p = w.p;
    a.y = y;
    a.h = h;
    a.M = M;
    a.d = d;
    a.I = blk->I;
    a.eps = eps;
    a.bar = bar;
    a.status = status_word();
    if (a.status != nullptr && decode_block_supported(a, dt)) {
      MMF_CUDA(timed("decode_block", s, [&] { return launch_decode_block(a, dt, s); }), "decode block");
      return MMF_OK;
    }
  }
  TGemmArgs tm = gemm_args(fcg, 3, w.qa.q, w.qa.s, w.qa.qsum, M, w.og, d, nullptr, nullptr);
  for (int i = 0; i < 3; ++i) tm.wu[i] = blk->wu[i];
  const bool fused_mixer = T > 1 && fused_mlgru_enabled() && gemm_uses_tc(tm, Epi::kStore) &&
                           tgemm_tc_mlgru_supported(tm, T, d);
  // prefill: the scan's scratch (all-ones before the scan) is filled by the
  // quantiser of x as side work, so no memset sits between the kernels
  const size_t scan_fill = fused_mixer ? tgemm_tc_mlgru_ws_bytes(B, T, d) : (T > 1 ? mlgru_scan_ws_bytes(B, T, d) : 0);
  // token mixer: x quantised once for f, c, g (shared gain)
  if (fused_mixer) {
    MMF_CUDA(timed("rmsnorm_quant", s,
                   [&] {
                     return launch_rmsnorm_quant(x, dt, M, d, W.f.gain, eps, w.qa.q, w.qa.s, w.qa.qsum, status_word(),
                                                 s, w.scan, scan_fill);
                   }),
             "block quant x");
    int* status = nullptr;
    mmf_status r = device_status_ptr(&status);
    if (r != MMF_OK) return r;
    MMF_CUDA(timed("tgemm_tc_mlgru", s, [&] { return launch_tgemm_tc_mlgru(tm, dt, T, d, h, w.scan, status, s); }),
             "block fcg+mlgru");
  } else if (T == 1) {
    // decode: projections and one recurrence step in one launch; h updated in place
    TGemmArgs a = gemm_args(fcg, 3, w.qa.q, w.qa.s, w.qa.qsum, M, w.og, d, nullptr, h);
    mmf_status r = quant_gemm(x, W.f.gain, eps, w.qa, a, Epi::kScanStep, dt, s, "fcg_step", false);
    if (r != MMF_OK) return r;
  } else {
    TGemmArgs a = gemm_args(fcg, 3, w.qa.q, w.qa.s, w.qa.qsum, M, w.pre, 3 * d, nullptr, nullptr);
    for (int i = 0; i < 3; ++i) a.wu[i] = blk->wu[i];
    mmf_status r = quant_gemm(x, W.f.gain, eps, w.qa, a, Epi::kStore, dt, s, "fcg", false, w.scan, scan_fill);
    if (r != MMF_OK) return r;
    int* status = nullptr;
    r = device_status_ptr(&status);
    if (r != MMF_OK) return r;
    MMF_CUDA(timed("mlgru_scan", s, [&] { return launch_mlgru_scan(w.pre, dt, B, T, d, h, w.og, w.scan, status, s); }),
             "block scan");
  }
  const mmf_tlinear* op[1] = {&W.o};
  TGemmArgs b = gemm_args(op, 1, w.qa.q, w.qa.s, w.qa.qsum, M, w.y1, d, x, nullptr);
  b.wu[0] = blk->wu[3];
  mmf_status r = quant_gemm(w.og, W.o.gain, eps, w.qa, b, Epi::kStore, dt, s, "o", false);
  if (r != MMF_OK) return r;
  // channel mixer
  return run_glu(&W.gate, &W.up, &W.down, w.y1, w.y1, y, M, dt, eps, w.p, w.qa, s, blk->wu + 4);
}

mmf_status check_forward_args(const mmf_block* blk, mmf_state* st, const void* x, void* y, int B, int T,
                              mmf_dtype dt, float eps, void* ws, const char* who) {
  if (!blk || !st) return fail(MMF_ERR_INVALID_ARG, "%s: null block/state", who);
  if (!dtype_ok(dt)) return fail(MMF_ERR_INVALID_ARG, "%s: bad dtype", who);
  if (B < 1 || T < 0) return fail(MMF_ERR_INVALID_ARG, "%s: B=%d T=%d", who, B, T);
  if (!(eps > 0.0f)) return fail(MMF_ERR_INVALID_ARG, "%s: eps must be > 0", who);
  if (B != st->B || blk->d != st->d)
    return fail(MMF_ERR_UNSUPPORTED_SHAPE, "%s: state is B=%d d=%d, call has B=%d d=%d", who, st->B, st->d, B, blk->d);
  if (T == 0) return MMF_OK;
  if (!x || !y || !ws) return fail(MMF_ERR_INVALID_ARG, "%s: null x/y/ws", who);
  if (!aligned16(x) || !aligned16(y) || !aligned16(ws)) return fail(MMF_ERR_MISALIGNED, "%s: pointer alignment", who);
  const size_t e = elem_bytes(dt);
  const char* xb = static_cast<const char*>(x);
  const char* yb = static_cast<const char*>(y);
  const size_t n = (size_t)B * T * blk->d * e;
  if (xb < yb + n && yb < xb + n) return fail(MMF_ERR_INVALID_ARG, "%s: x and y overlap", who);
  return MMF_OK;
}

}  // namespace

extern "C" size_t mmf_block_ws_size(const mmf_block* blk, int32_t B, int32_t T) {
  if (!blk || B < 0 || T < 0) return 0;
  return carve_block(nullptr, B, T, blk->d, blk->I, MMF_F32).bytes;
}

extern "C" mmf_status mmf_block_forward(const mmf_block* blk, int32_t layer, mmf_state* st, const void* x, void* y,
                                        int32_t B, int32_t T, mmf_dtype dtype, float eps, void* ws, size_t ws_bytes,
                                        void* stream) {
  mmf_status r = check_forward_args(blk, st, x, y, B, T, dtype, eps, ws, "mmf_block_forward");
  if (r != MMF_OK) return r;
  if (layer < 0 || layer >= st->L) return fail(MMF_ERR_INVALID_ARG, "mmf_block_forward: layer %d of %d", layer, st->L);
  if (T == 0) return MMF_OK;
  BlockWs w = carve_block(ws, B, T, blk->d, blk->I, dtype);
  if (ws_bytes < mmf_block_ws_size(blk, B, T))
    return fail(MMF_ERR_WORKSPACE, "mmf_block_forward: ws_bytes=%zu < %zu", ws_bytes, mmf_block_ws_size(blk, B, T));
  return block_forward_impl(blk, mmf_state_layer(st, layer), st->bar, x, y, B, T, dtype, eps, w, as_stream(stream));
}

extern "C" mmf_status mmf_stack_forward(const mmf_block* const* blocks, int32_t L, mmf_state* st, const void* x,
                                        void* y, int32_t B, int32_t T, mmf_dtype dtype, float eps, void* ws,
                                        size_t ws_bytes, void* stream) {
  if (!blocks || L < 1) return fail(MMF_ERR_INVALID_ARG, "mmf_stack_forward: blocks=%p L=%d", (void*)blocks, L);
  if (!st || L > st->L) return fail(MMF_ERR_INVALID_ARG, "mmf_stack_forward: state has fewer than %d layers", L);
  size_t need = 0;
  for (int l = 0; l < L; ++l) {
    mmf_status r = check_forward_args(blocks[l], st, x, y, B, T, dtype, eps, ws, "mmf_stack_forward");
    if (r != MMF_OK) return r;
    if (blocks[l]->d != blocks[0]->d)
      return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_stack_forward: block %d has d=%d", l, blocks[l]->d);
    need = std::max(need, mmf_block_ws_size(blocks[l], B, T));
  }
  if (T == 0) return MMF_OK;
  if (ws_bytes < need) return fail(MMF_ERR_WORKSPACE, "mmf_stack_forward: ws_bytes=%zu < %zu", ws_bytes, need);
  cudaStream_t s = as_stream(stream);
  const void* cur = x;
  for (int l = 0; l < L; ++l) {
    BlockWs w = carve_block(ws, B, T, blocks[l]->d, blocks[l]->I, dtype);
    void* dst = (l == L - 1) ? y : ((l % 2 == 0) ? w.ping : w.pong);
    mmf_status r = block_forward_impl(blocks[l], mmf_state_layer(st, l), st->bar, cur, dst, B, T, dtype, eps, w, s);
    if (r != MMF_OK) return r;
    cur = dst;
  }
  return MMF_OK;
}

// ------------------------------------------------------------------ launch timing ABI

extern "C" mmf_status mmf_prof_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  return MMF_OK;
}

extern "C" int32_t mmf_prof_collect(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (const ProfPair& p : g_prof_pending) {
    cudaError_t e = cudaEventSynchronize(p.b);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, p.a, p.b);
    if (e != cudaSuccess) {
      cuda_fail(e, "mmf_prof_collect");
      return -1;
    }
    g_prof_kinds[p.kind].launches += 1;
    g_prof_kinds[p.kind].ms += ms;
    g_prof_free.push_back(p.a);
    g_prof_free.push_back(p.b);
  }
  g_prof_pending.clear();
  return (int32_t)g_prof_kinds.size();
}

extern "C" mmf_status mmf_prof_get(int32_t i, char* name, size_t name_len, int64_t* launches, double* total_ms) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (i < 0 || i >= (int32_t)g_prof_kinds.size()) return fail(MMF_ERR_INVALID_ARG, "mmf_prof_get: index %d", i);
  const ProfKind& k = g_prof_kinds[i];
  if (name && name_len > 0) {
    strncpy(name, k.name.c_str(), name_len - 1);
    name[name_len - 1] = '\0';
  }
  if (launches) *launches = k.launches;
  if (total_ms) *total_ms = k.ms;
  return MMF_OK;
}

extern "C" void mmf_prof_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (const ProfPair& p : g_prof_pending) {
    g_prof_free.push_back(p.a);
    g_prof_free.push_back(p.b);
  }
  g_prof_pending.clear();
  g_prof_kinds.clear();
}
