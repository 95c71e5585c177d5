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

// Contraction dispatch: the tcgen05 kernel from 128 tokens, the mma.sync
// kernel for decode-sized token counts and for shapes the tcgen05 kernel does
// not take. MMF_GEMM_PATH=mma|tc|auto (default auto) pins one implementation;
// both compute the same exact integer accumulators.
constexpr int kTcMinTokens = 128;

int gemm_path_pref() {
  const char* e = getenv("MMF_GEMM_PATH");
  if (e == nullptr) return 0;
  if (strcmp(e, "mma") == 0) return 1;
  if (strcmp(e, "tc") == 0) return 2;
  return 0;
}

// Below 128 tokens the tcgen05 kernel still wins on wide projections, whose
// 128 x 256 tiles (one, half empty, per 256 output columns) keep enough SMs
// busy: 2.7B decode at 64 sequences, gate|up (54 tiles) 1.31 -> 0.66 ms per
// step, at 32 sequences 0.78 -> 0.65 ms; the o and down projections (10
// tiles) and anything at 16 sequences stay faster on the mma.sync kernel.
constexpr int kTcMinTokensWide = 32;
constexpr int kTcMinTilesWide = 48;

bool gemm_uses_tc(const TGemmArgs& a, Epi epi) {
  const int pref = gemm_path_pref();
  if (!tgemm_tc_supported(a, epi) || pref == 1) return false;
  if (pref >= 2 || a.M >= kTcMinTokens) return true;
  const int cols = epi == Epi::kGlu ? a.N / 128 : ceil_div(a.nseg * a.N, 256);
  return a.M >= kTcMinTokensWide && cols >= kTcMinTilesWide;
}

// Whether the decode contraction quantises its own token rows (both ways give
// the same codes). Every CTA then repeats the row work, which on one B200 beat
// the standalone quantiser plus one kernel boundary only for single-token
// calls (1.3B decode at 4 tokens: 0.69 ms per step fused, 0.59 ms split).
// MMF_DECODE_FUSED_QUANT=1 fuses whenever the shapes allow, =0 never.
// Single-token calls quantise inside the contraction unless the projection is
// so wide (more than 4 16-row CTAs per SM, e.g. a 32000-entry LM head) that
// every CTA quantising the same row costs more than one quantiser launch
// (2560 -> 32000: 32.8 us fused, 19.5 us with the quantiser). Up to 4 tokens
// they do so when the projection is one wave of CTAs (single calls 2048 ->
// 2048 at 4 tokens: 3.90 vs 4.54 us; 5632 -> 2048: 6.78 vs 7.47 us); at 16
// tokens, or on wider outputs (2048 -> 5632), the separate quantiser is faster.
bool decode_fused_quant_wanted(int M, int N) {
  const char* e = getenv("MMF_DECODE_FUSED_QUANT");
  if (e != nullptr && strcmp(e, "1") == 0) return true;
  if (e != nullptr && strcmp(e, "0") == 0) return false;
  if (M == 1) return ceil_div(N, 16) <= 4 * num_sms();
  return M <= 4 && ceil_div(N, 16) <= num_sms();
}

// `what` names the projection for the launch-timing totals ("fcg", "o", ...).
cudaError_t run_gemm(const TGemmArgs& a, Epi epi, mmf_dtype dt, cudaStream_t s, const char* what = "") {
  const bool use_tc = gemm_uses_tc(a, epi);
  char name[48];
  snprintf(name, sizeof(name), "%s%s%s", use_tc ? "tgemm_tc" : "tgemm_mma", what[0] ? ":" : "", what);
  if (use_tc) {
    int* st = nullptr;
    if (device_status_ptr(&st) != MMF_OK) return cudaErrorUnknown;
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
  if (!gemm_uses_tc(a, epi) && decode_fused_quant_wanted(a.M, a.N) &&
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

// Blocks make one-byte copies of their codes for the prefill contraction
// (4x the packed weight memory), at their first prefill-sized call, unless
// MMF_PREFILL_UNPACKED=0.
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
// ddesc: device copy of the block's decode descriptor (weights, scales,
// biases, gains), read by the one-launch decode step.
// wu: the one-byte codes the prefill contraction loads (the caller's, or the
// library's copies in owned, made by the first prefill-sized call; null: the
// contraction expands the packed codes). codes_tried and mu guard that copy.
struct mmf_block {
  mmf_block_weights w;
  int d, I;
  mutable const uint8_t* wu[7];
  mutable uint8_t* owned[7];
  mutable bool codes_tried;
  mutable std::mutex mu;
  DecodeLayerDesc* ddesc;
};

// xbuf: exchange buffers of the one-launch decode step, allocated by the first
// decode step that needs them: a header of L launch-parity words and one abort
// word (rounded up to 256 bytes), then decode_xlayer_bytes(B, d, xI) bytes per
// layer, filled with all-ones bytes. xdt is the dtype of the last decode step.
struct mmf_state {
  float* h;
  int L, B, d;
  uint8_t* xbuf;
  size_t xbytes;
  int xI, xdt;
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
    if (v == 8)
      return fail(MMF_ERR_INVALID_ARG, "a token id was outside [0, V); its embedding row was written as zeros");
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
  MMF_CUDA(timed("mlgru_scan", s, [&] { return launch_mlgru_scan(pre, dtype, B, T, d, h, o, status, s); }),
           "mlgru_scan");
  return MMF_OK;
}

extern "C" size_t mmf_mlgru_scan_backward_ws_size(int32_t B, int32_t T, int32_t d) {
  if (B < 0 || T < 0 || d < 0) return 0;
  return mlgru_scan_bwd_ws_bytes(B, T, d);
}

extern "C" mmf_status mmf_mlgru_scan_states(const void* pre, mmf_dtype dtype, int32_t B, int32_t T, int32_t d,
                                            float* h, void* o, float* hs, void* stream) {
  if (!dtype_ok(dtype)) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan_states: bad dtype");
  if (B < 0 || T < 0 || d < 1) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan_states: B=%d T=%d d=%d", B, T, d);
  if (d % 8 != 0) return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_mlgru_scan_states: d=%d %% 8 != 0", d);
  if (B == 0 || T == 0) return MMF_OK;
  if (!pre || !h || !hs) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan_states: null pointer");
  if (!aligned16(pre) || !aligned16(h) || !aligned16(hs) || (o && !aligned16(o)))
    return fail(MMF_ERR_MISALIGNED, "mmf_mlgru_scan_states");
  cudaStream_t s = as_stream(stream);
  int* status = nullptr;
  mmf_status r = device_status_ptr(&status);
  if (r != MMF_OK) return r;
  MMF_CUDA(timed("mlgru_scan_states", s,
                 [&] { return launch_mlgru_scan_states(pre, dtype, B, T, d, h, o, hs, status, s); }),
           "mlgru_scan_states");
  return MMF_OK;
}

extern "C" mmf_status mmf_mlgru_scan_backward(const void* pre, mmf_dtype dtype, int32_t B, int32_t T, int32_t d,
                                              const float* h0, const void* dout, const float* dhT, const float* hs,
                                              void* dpre, float* dh0, void* ws, size_t ws_bytes, void* stream) {
  if (!dtype_ok(dtype)) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan_backward: bad dtype");
  if (B < 0 || T < 0 || d < 1) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan_backward: B=%d T=%d d=%d", B, T, d);
  if (d % 8 != 0) return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_mlgru_scan_backward: d=%d %% 8 != 0", d);
  if (B == 0 || T == 0) return MMF_OK;
  if (!pre || !h0 || !dout || !dpre || !dh0 || (!hs && !ws))
    return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan_backward: null pointer");
  if (!aligned16(pre) || !aligned16(h0) || !aligned16(dout) || !aligned16(dpre) || !aligned16(dh0) ||
      (ws && !aligned16(ws)) || (dhT && !aligned16(dhT)) || (hs && !aligned16(hs)))
    return fail(MMF_ERR_MISALIGNED, "mmf_mlgru_scan_backward");
  if (!hs && ws_bytes < mlgru_scan_bwd_ws_bytes(B, T, d))
    return fail(MMF_ERR_WORKSPACE, "mmf_mlgru_scan_backward: ws_bytes=%zu < %zu", ws_bytes,
                mlgru_scan_bwd_ws_bytes(B, T, d));
  const char* hb = reinterpret_cast<const char*>(h0);
  const char* db = reinterpret_cast<const char*>(dh0);
  const size_t sb = sizeof(float) * (size_t)B * d;
  if (hb < db + sb && db < hb + sb) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan_backward: h0 and dh0 overlap");
  cudaStream_t s = as_stream(stream);
  int* status = nullptr;
  mmf_status r = device_status_ptr(&status);
  if (r != MMF_OK) return r;
  MMF_CUDA(timed("mlgru_scan_backward", s,
                 [&] { return launch_mlgru_scan_bwd(pre, dtype, B, T, d, h0, dout, dhT, hs, dpre, dh0, ws, status, s); }),
           "mlgru_scan_backward");
  return MMF_OK;
}

extern "C" size_t mmf_mlgru_scan_gnorm_ws_size(int32_t B, int32_t T, int32_t d) {
  if (B < 0 || T < 0 || d < 0) return 0;
  return mlgru_scan_gnorm_ws_bytes(B, T, d);
}

extern "C" mmf_status mmf_mlgru_scan_gnorm(const void* pre, mmf_dtype dtype, int32_t B, int32_t T, int32_t d,
                                           float* h, const float* gain, float eps, void* o, void* ws,
                                           size_t ws_bytes, void* stream) {
  if (!dtype_ok(dtype)) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan_gnorm: bad dtype");
  if (B < 0 || T < 0 || d < 1) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan_gnorm: B=%d T=%d d=%d", B, T, d);
  if (!(eps > 0.0f)) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan_gnorm: eps must be > 0");
  if (d % 8 != 0) return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_mlgru_scan_gnorm: d=%d %% 8 != 0", d);
  if (B == 0 || T == 0) return MMF_OK;
  if (!pre || !h || !gain || !o || !ws) return fail(MMF_ERR_INVALID_ARG, "mmf_mlgru_scan_gnorm: null pointer");
  if (!aligned16(pre) || !aligned16(h) || !aligned16(gain) || !aligned16(o) || !aligned16(ws))
    return fail(MMF_ERR_MISALIGNED, "mmf_mlgru_scan_gnorm");
  if (ws_bytes < mlgru_scan_gnorm_ws_bytes(B, T, d))
    return fail(MMF_ERR_WORKSPACE, "mmf_mlgru_scan_gnorm: ws_bytes=%zu < %zu", ws_bytes,
                mlgru_scan_gnorm_ws_bytes(B, T, d));
  cudaStream_t s = as_stream(stream);
  int* status = nullptr;
  mmf_status r = device_status_ptr(&status);
  if (r != MMF_OK) return r;
  MMF_CUDA(timed("mlgru_scan_gnorm", s,
                 [&] { return launch_mlgru_scan_gnorm(pre, dtype, B, T, d, h, gain, eps, o, ws, status, s); }),
           "mlgru_scan_gnorm");
  return MMF_OK;
}

// ------------------------------------------------------------------ model ends

extern "C" mmf_status mmf_embed(const int32_t* ids, int32_t M, const void* table, int32_t V, int32_t d,
                                mmf_dtype dtype, void* x, void* stream) {
  if (!dtype_ok(dtype)) return fail(MMF_ERR_INVALID_ARG, "mmf_embed: bad dtype");
  if (M < 0 || V < 1 || d < 1) return fail(MMF_ERR_INVALID_ARG, "mmf_embed: M=%d V=%d d=%d", M, V, d);
  if (d % 16 != 0) return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_embed: d=%d %% 16 != 0", d);
  if (M == 0) return MMF_OK;
  if (!ids || !table || !x) return fail(MMF_ERR_INVALID_ARG, "mmf_embed: null pointer");
  if (!aligned16(table) || !aligned16(x)) return fail(MMF_ERR_MISALIGNED, "mmf_embed");
  int* status = nullptr;
  mmf_status r = device_status_ptr(&status);
  if (r != MMF_OK) return r;
  cudaStream_t s = as_stream(stream);
  MMF_CUDA(timed("embed", s, [&] { return launch_embed(ids, M, table, V, d, dtype, x, status, s); }), "embed");
  return MMF_OK;
}

extern "C" mmf_status mmf_argmax(const void* logits, mmf_dtype dtype, int32_t M, int32_t V, int32_t* ids,
                                 void* stream) {
  if (!dtype_ok(dtype)) return fail(MMF_ERR_INVALID_ARG, "mmf_argmax: bad dtype");
  if (M < 0 || V < 1) return fail(MMF_ERR_INVALID_ARG, "mmf_argmax: M=%d V=%d", M, V);
  if (M == 0) return MMF_OK;
  if (!logits || !ids) return fail(MMF_ERR_INVALID_ARG, "mmf_argmax: null pointer");
  cudaStream_t s = as_stream(stream);
  MMF_CUDA(timed("argmax", s, [&] { return launch_argmax(logits, dtype, M, V, ids, s); }), "argmax");
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
mmf_status dbg_codes(const mmf_block_debug* dbg, int i, const QAct& qa, int M, int K, cudaStream_t s);

mmf_status run_glu(const mmf_tlinear* gate, const mmf_tlinear* up, const mmf_tlinear* down, const void* x,
                   const void* residual, void* y, int M, mmf_dtype dt, float eps, void* p, const QAct& qa,
                   cudaStream_t s, const uint8_t* const* wu = nullptr /* gate, up, down one-byte codes */,
                   const mmf_block_debug* dbg = nullptr) {
  const mmf_tlinear* gu[2] = {gate, up};
  TGemmArgs a = gemm_args(gu, 2, qa.q, qa.s, qa.qsum, M, p, gate->N, nullptr, nullptr);
  if (wu) {
    a.wu[0] = wu[0];
    a.wu[1] = wu[1];
  }   // otherwise the layers' own codes (if any), set by gemm_args
  mmf_status r = quant_gemm(x, gate->gain, eps, qa, a, Epi::kGlu, dt, s, "gate_up", dbg != nullptr);
  if (r == MMF_OK) r = dbg_codes(dbg, 2, qa, M, gate->K, s);
  if (r != MMF_OK) return r;
  const mmf_tlinear* dn[1] = {down};
  TGemmArgs b = gemm_args(dn, 1, qa.q, qa.s, qa.qsum, M, y, down->N, residual, nullptr);
  if (wu) b.wu[0] = wu[2];
  r = quant_gemm(p, down->gain, eps, qa, b, Epi::kStore, dt, s, "down", dbg != nullptr);
  if (r == MMF_OK) r = dbg_codes(dbg, 3, qa, M, down->K, s);
  return r;
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
  if (w->gnorm != nullptr && !aligned16(w->gnorm)) return fail(MMF_ERR_MISALIGNED, "mmf_block_create: gnorm");
  if ((st = check_glu(&w->gate, &w->up, &w->down, d)) != MMF_OK) return st;
  if (w->gate.N != I) return fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_block_create: gate N=%d != I=%d", w->gate.N, I);
  mmf_block* b = new (std::nothrow) mmf_block;
  if (!b) return fail(MMF_ERR_NOMEM, "mmf_block_create: out of host memory");
  b->w = *w;
  b->d = d;
  b->I = I;
  b->ddesc = nullptr;
  b->codes_tried = false;
  const mmf_tlinear* all[7] = {&w->f, &w->c, &w->g, &w->o, &w->gate, &w->up, &w->down};
  for (int i = 0; i < 7; ++i) {
    b->wu[i] = all[i]->codes;
    b->owned[i] = nullptr;
  }
  {   // the decode step's device descriptor of this block
    DecodeLayerDesc h{};
    for (int i = 0; i < 7; ++i) {
      h.w[i] = all[i]->packed;
      h.gamma[i] = all[i]->gamma;
      h.bias[i] = all[i]->bias;
    }
    h.gain[0] = w->f.gain;
    h.gain[1] = w->o.gain;
    h.gain[2] = w->gate.gain;
    h.gain[3] = w->down.gain;
    // without it the block's decode steps take the four-contraction path
    cudaError_t e = cudaMalloc(&b->ddesc, sizeof(DecodeLayerDesc));
    if (e == cudaSuccess) e = cudaMemcpy(b->ddesc, &h, sizeof(h), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      cudaFree(b->ddesc);
      b->ddesc = nullptr;
    }
  }
  *out = b;
  return MMF_OK;
}

extern "C" void mmf_block_destroy(mmf_block* blk) {
  if (!blk) return;
  for (int i = 0; i < 7; ++i) cudaFree(blk->owned[i]);
  cudaFree(blk->ddesc);
  delete blk;
}

extern "C" mmf_status mmf_block_release_codes(mmf_block* blk) {
  if (!blk) return fail(MMF_ERR_INVALID_ARG, "mmf_block_release_codes: null block");
  std::lock_guard<std::mutex> lock(blk->mu);
  bool any = false;
  for (int i = 0; i < 7; ++i) any = any || blk->owned[i] != nullptr;
  if (any) MMF_CUDA(cudaDeviceSynchronize(), "mmf_block_release_codes: synchronize");
  const mmf_tlinear* all[7] = {&blk->w.f, &blk->w.c, &blk->w.g, &blk->w.o, &blk->w.gate, &blk->w.up, &blk->w.down};
  for (int i = 0; i < 7; ++i) {
    if (blk->owned[i] != nullptr) MMF_CUDA(cudaFree(blk->owned[i]), "mmf_block_release_codes: cudaFree");
    blk->owned[i] = nullptr;
    blk->wu[i] = all[i]->codes;   // the caller's own one-byte codes, if it gave any
  }
  blk->codes_tried = false;   // the next prefill-sized call makes the copy again
  return MMF_OK;
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
  e = cudaMemset(st->h, 0, bytes);
  if (e != cudaSuccess) {
    cudaFree(st->h);
    delete st;
    return cuda_fail(e, "mmf_state_create: cudaMemset");
  }
  st->L = L;
  st->B = B;
  st->d = d;
  st->xbuf = nullptr;
  st->xbytes = 0;
  st->xI = 0;
  st->xdt = -1;
  *out = st;
  return MMF_OK;
}

extern "C" void mmf_state_destroy(mmf_state* st) {
  if (!st) return;
  cudaFree(st->h);
  cudaFree(st->xbuf);
  delete st;
}

namespace {

size_t decode_header_bytes(int L) { return round_up(sizeof(uint32_t) * ((size_t)L + 1), 256); }

// Launch parities all zero, abort word zero, every exchange element all-ones.
cudaError_t reset_decode_buffers(mmf_state* st, cudaStream_t s) {
  if (st->xbuf == nullptr) return cudaSuccess;
  const size_t hb = decode_header_bytes(st->L);
  cudaError_t e = cudaMemsetAsync(st->xbuf, 0, hb, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(st->xbuf + hb, 0xff, st->xbytes - hb, s);
  return e;
}

// Exchange buffers for decode steps of blocks with inner size I in dtype dt:
// allocated (cudaMalloc) the first time and whenever a larger I comes, and
// reset when the dtype changes.
mmf_status ensure_decode_buffers(mmf_state* st, int I, mmf_dtype dt, cudaStream_t s) {
  if (st->xbuf == nullptr || I > st->xI) {
    const size_t bytes = decode_header_bytes(st->L) + (size_t)st->L * decode_xlayer_bytes(st->B, st->d, I);
    if (st->xbuf != nullptr) {
      MMF_CUDA(cudaStreamSynchronize(s), "decode buffers: synchronise");
      cudaFree(st->xbuf);
      st->xbuf = nullptr;
    }
    uint8_t* p = nullptr;
    cudaError_t e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) return fail(MMF_ERR_NOMEM, "decode buffers: cudaMalloc(%zu): %s", bytes, cudaGetErrorString(e));
    st->xbuf = p;
    st->xbytes = bytes;
    st->xI = I;
    st->xdt = -1;
  }
  if (st->xdt != (int)dt) {
    MMF_CUDA(reset_decode_buffers(st, s), "decode buffers: reset");
    st->xdt = (int)dt;
  }
  return MMF_OK;
}

}  // namespace

extern "C" mmf_status mmf_state_reset(mmf_state* st, void* stream) {
  if (!st) return fail(MMF_ERR_INVALID_ARG, "mmf_state_reset: null state");
  MMF_CUDA(cudaMemsetAsync(st->h, 0, sizeof(float) * (size_t)st->L * st->B * st->d, as_stream(stream)),
           "mmf_state_reset");
  MMF_CUDA(reset_decode_buffers(st, as_stream(stream)), "mmf_state_reset: decode buffers");
  return MMF_OK;
}

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
  void* og;    // [M, d] o' (the scan's output gate applied)
  void* gn;    // g_norm blocks: the scan's scratch (mlgru_scan_gnorm_ws_bytes), else null
  void* y1;    // [M, d] after the token mixer
  void* p;     // [M, I] GLU product
  void* ping;  // [M, d] stack intermediates
  void* pong;
  size_t bytes;
};

BlockWs carve_block(void* base, int B, int T, int d, int I, mmf_dtype dt, bool gnorm) {
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
  w.gn = gnorm ? c.take<char>(mlgru_scan_gnorm_ws_bytes(B, T, d)) : nullptr;
  w.bytes = c.off + 256;
  return w;
}

// Decode steps (T = 1) of up to 8 sequences run as one launch over all the
// layers of the call (decode_step.cu) unless MMF_DECODE_STEP_KERNEL=0, which
// selects the four contractions per block instead (the same arithmetic; the
// codes can differ only where the fp64 sum of squares rounds differently).
bool decode_step_enabled() {
  const char* e = getenv("MMF_DECODE_STEP_KERNEL");
  return e == nullptr || strcmp(e, "0") != 0;
}


bool decode_step_usable(const mmf_block* const* blocks, int L, int B, mmf_dtype dt) {
  if (!decode_step_enabled()) return false;
  for (int l = 0; l < L; ++l)
    if (blocks[l]->I != blocks[0]->I || blocks[l]->d != blocks[0]->d || blocks[l]->ddesc == nullptr ||
        blocks[l]->w.gnorm != nullptr)
      return false;
  return decode_step_supported(B, blocks[0]->d, blocks[0]->I, std::min(L, kDecodeMaxLayers), dt);
}

// One decode step of blocks[0 .. L) (state layers layer0 ..), in launches of
// at most kDecodeMaxLayers layers; x -> y, `mid` [B, d] carries the output of
// one launch to the next.
mmf_status run_decode_step(const mmf_block* const* blocks, int L, int layer0, mmf_state* st, const void* x, void* y,
                           void* mid, int B, mmf_dtype dt, float eps, cudaStream_t s, const mmf_block_debug* dbg) {
  mmf_status r = ensure_decode_buffers(st, blocks[0]->I, dt, s);
  if (r != MMF_OK) return r;
  int* status = nullptr;
  if ((r = device_status_ptr(&status)) != MMF_OK) return r;
  const size_t hb = decode_header_bytes(st->L);
  for (int l0 = 0; l0 < L; l0 += kDecodeMaxLayers) {
    const int n = std::min(kDecodeMaxLayers, L - l0);
    DecodeStepArgs a{};
    for (int l = 0; l < n; ++l) a.layer[l] = blocks[l0 + l]->ddesc;
    a.x = l0 == 0 ? x : mid;
    a.y = l0 + n == L ? y : mid;
    a.h = st->h;
    a.xbuf = st->xbuf + hb;
    a.parity = reinterpret_cast<unsigned*>(st->xbuf);
    a.abort_word = reinterpret_cast<int*>(st->xbuf) + st->L;
    a.status = status;
    if (dbg != nullptr && n == 1) a.dbg = *dbg;
    a.wait_cycles = wait_limit_cycles();
    a.eps = eps;
    a.L = n;
    a.layer0 = layer0 + l0;
    a.M = B;
    a.d = blocks[0]->d;
    a.I = blocks[0]->I;
    a.xI = st->xI;
    a.skip_cta = test_hook("MMF_DECODE_SKIP_CTA");   // test: CTA b never publishes its first stage
    MMF_CUDA(timed("decode_step", s, [&] { return launch_decode_step(a, dt, s); }), "decode step");
  }
  return MMF_OK;
}

// Stream-ordered copy of the quantised input of stage i (codes, scales) into the debug outputs.
mmf_status dbg_codes(const mmf_block_debug* dbg, int i, const QAct& qa, int M, int K, cudaStream_t s) {
  if (dbg == nullptr) return MMF_OK;
  if (dbg->q[i]) MMF_CUDA(cudaMemcpyAsync(dbg->q[i], qa.q, (size_t)M * K, cudaMemcpyDeviceToDevice, s), "dbg q");
  if (dbg->scale[i])
    MMF_CUDA(cudaMemcpyAsync(dbg->scale[i], qa.s, sizeof(float) * M, cudaMemcpyDeviceToDevice, s), "dbg scale");
  return MMF_OK;
}

mmf_status dbg_copy(void* dst, const void* src, size_t bytes, cudaStream_t s) {
  if (dst == nullptr) return MMF_OK;
  MMF_CUDA(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s), "dbg copy");
  return MMF_OK;
}

// The block's one-byte code copies, made once, by the first call with enough
// tokens for the tensor-core contraction: allocated with cudaMalloc and filled
// by one kernel on the call's stream (so the contraction, later on the same
// stream, sees them). Without device memory for all of them the block keeps the
// packed codes (same results).
void ensure_prefill_codes(const mmf_block* b, cudaStream_t s) {
  std::lock_guard<std::mutex> lock(b->mu);
  if (b->codes_tried) return;
  b->codes_tried = true;
  if (!prefill_unpacked_enabled()) return;
  const mmf_block_weights& w = b->w;
  const mmf_tlinear* all[7] = {&w.f, &w.c, &w.g, &w.o, &w.gate, &w.up, &w.down};
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
    return;
  }
  for (int i = 0; i < 7; ++i) {
    if (b->owned[i] == nullptr) continue;
    if (launch_unpack_codes(all[i]->packed, all[i]->N, all[i]->K, b->owned[i], s) != cudaSuccess) {
      (void)cudaGetLastError();
      return;   // this and later matrices keep their packed codes
    }
    b->wu[i] = b->owned[i];
  }
}

mmf_status block_forward_impl(const mmf_block* blk, float* h, const void* x, void* y, int B, int T, mmf_dtype dt,
                              float eps, const BlockWs& w, cudaStream_t s, const mmf_block_debug* dbg = nullptr) {
  const int M = B * T, d = blk->d;
  const mmf_block_weights& W = blk->w;
  const mmf_tlinear* fcg[3] = {&W.f, &W.c, &W.g};
  const bool want = dbg != nullptr;
  const bool gnorm = W.gnorm != nullptr;
  if (T > 1 && (M >= kTcMinTokens || gemm_path_pref() >= 2)) ensure_prefill_codes(blk, s);
  // token mixer: x quantised once for f, c, g (shared gain)
  if (T == 1 && !gnorm) {
    // decode: projections and one recurrence step in one launch; h updated in place
    TGemmArgs a = gemm_args(fcg, 3, w.qa.q, w.qa.s, w.qa.qsum, M, w.og, d, nullptr, h);
    if (want) a.pre_out = dbg->pre;
    mmf_status r = quant_gemm(x, W.f.gain, eps, w.qa, a, Epi::kScanStep, dt, s, "fcg_step", want);
    if (r == MMF_OK) r = dbg_codes(dbg, 0, w.qa, M, d, s);
    if (r != MMF_OK) return r;
  } else {
    TGemmArgs a = gemm_args(fcg, 3, w.qa.q, w.qa.s, w.qa.qsum, M, w.pre, 3 * d, nullptr, nullptr);
    for (int i = 0; i < 3; ++i) a.wu[i] = blk->wu[i];
    mmf_status r = quant_gemm(x, W.f.gain, eps, w.qa, a, Epi::kStore, dt, s, "fcg", want);
    if (r == MMF_OK) r = dbg_codes(dbg, 0, w.qa, M, d, s);
    if (r == MMF_OK && want) r = dbg_copy(dbg->pre, w.pre, (size_t)M * 3 * d * elem_bytes(dt), s);
    if (r != MMF_OK) return r;
    int* status = nullptr;
    r = device_status_ptr(&status);
    if (r != MMF_OK) return r;
    if (gnorm)   // scan, then o' formed and quantised for the o projection in one row kernel
      MMF_CUDA(timed("mlgru_scan_gnorm", s,
                     [&] {
                       return launch_mlgru_scan_gnorm_quant(w.pre, dt, B, T, d, h, W.gnorm, eps, want ? w.og : nullptr,
                                                            w.gn, status, W.o.gain, eps, w.qa.q, w.qa.s, w.qa.qsum, s);
                     }),
               "block scan");
    else
      MMF_CUDA(timed("mlgru_scan", s, [&] { return launch_mlgru_scan(w.pre, dt, B, T, d, h, w.og, status, s); }),
               "block scan");
  }
  const mmf_tlinear* op[1] = {&W.o};
  TGemmArgs b = gemm_args(op, 1, w.qa.q, w.qa.s, w.qa.qsum, M, w.y1, d, x, nullptr);
  b.wu[0] = blk->wu[3];
  mmf_status r = MMF_OK;
  if (gnorm) {   // the codes of o' are already in w.qa
    MMF_CUDA(run_gemm(b, Epi::kStore, dt, s, "o"), "contraction");
  } else {
    r = quant_gemm(w.og, W.o.gain, eps, w.qa, b, Epi::kStore, dt, s, "o", want);
  }
  if (r == MMF_OK) r = dbg_codes(dbg, 1, w.qa, M, d, s);
  if (r != MMF_OK) return r;
  // channel mixer
  r = run_glu(&W.gate, &W.up, &W.down, w.y1, w.y1, y, M, dt, eps, w.p, w.qa, s, blk->wu + 4, dbg);
  if (r != MMF_OK || !want) return r;
  const size_t e = elem_bytes(dt);
  if ((r = dbg_copy(dbg->og, w.og, (size_t)M * d * e, s)) != MMF_OK) return r;
  if ((r = dbg_copy(dbg->y1, w.y1, (size_t)M * d * e, s)) != MMF_OK) return r;
  return dbg_copy(dbg->p, w.p, (size_t)M * blk->I * e, s);
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
  return carve_block(nullptr, B, T, blk->d, blk->I, MMF_F32, blk->w.gnorm != nullptr).bytes;
}

extern "C" mmf_status mmf_block_forward(const mmf_block* blk, int32_t layer, mmf_state* st, const void* x, void* y,
                                        int32_t B, int32_t T, mmf_dtype dtype, float eps, void* ws, size_t ws_bytes,
                                        void* stream) {
  mmf_status r = check_forward_args(blk, st, x, y, B, T, dtype, eps, ws, "mmf_block_forward");
  if (r != MMF_OK) return r;
  if (layer < 0 || layer >= st->L) return fail(MMF_ERR_INVALID_ARG, "mmf_block_forward: layer %d of %d", layer, st->L);
  if (T == 0) return MMF_OK;
  BlockWs w = carve_block(ws, B, T, blk->d, blk->I, dtype, blk->w.gnorm != nullptr);
  if (ws_bytes < mmf_block_ws_size(blk, B, T))
    return fail(MMF_ERR_WORKSPACE, "mmf_block_forward: ws_bytes=%zu < %zu", ws_bytes, mmf_block_ws_size(blk, B, T));
  if (T == 1 && decode_step_usable(&blk, 1, B, dtype))
    return run_decode_step(&blk, 1, layer, st, x, y, nullptr, B, dtype, eps, as_stream(stream), nullptr);
  return block_forward_impl(blk, mmf_state_layer(st, layer), x, y, B, T, dtype, eps, w, as_stream(stream));
}

extern "C" mmf_status mmf_block_forward_debug(const mmf_block* blk, int32_t layer, mmf_state* st, const void* x,
                                              void* y, int32_t B, int32_t T, mmf_dtype dtype, float eps, void* ws,
                                              size_t ws_bytes, void* stream, const mmf_block_debug* dbg) {
  if (dbg != nullptr) {
    const void* ptrs[12] = {dbg->pre, dbg->og, dbg->y1, dbg->p};
    for (int i = 0; i < 4; ++i) {
      ptrs[4 + i] = dbg->q[i];
      ptrs[8 + i] = dbg->scale[i];
    }
    for (const void* p : ptrs)
      if (p != nullptr && !aligned16(p)) return fail(MMF_ERR_MISALIGNED, "mmf_block_forward_debug: debug buffer");
  }
  mmf_status r = check_forward_args(blk, st, x, y, B, T, dtype, eps, ws, "mmf_block_forward_debug");
  if (r != MMF_OK) return r;
  if (layer < 0 || layer >= st->L)
    return fail(MMF_ERR_INVALID_ARG, "mmf_block_forward_debug: layer %d of %d", layer, st->L);
  if (T == 0) return MMF_OK;
  BlockWs w = carve_block(ws, B, T, blk->d, blk->I, dtype, blk->w.gnorm != nullptr);
  if (ws_bytes < mmf_block_ws_size(blk, B, T))
    return fail(MMF_ERR_WORKSPACE, "mmf_block_forward_debug: ws_bytes=%zu < %zu", ws_bytes,
                mmf_block_ws_size(blk, B, T));
  if (T == 1 && decode_step_usable(&blk, 1, B, dtype))
    return run_decode_step(&blk, 1, layer, st, x, y, nullptr, B, dtype, eps, as_stream(stream), dbg);
  return block_forward_impl(blk, mmf_state_layer(st, layer), x, y, B, T, dtype, eps, w, as_stream(stream), dbg);
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
  if (T == 1 && decode_step_usable(blocks, L, B, dtype)) {
    BlockWs w = carve_block(ws, B, T, blocks[0]->d, blocks[0]->I, dtype, false);
    return run_decode_step(blocks, L, 0, st, x, y, w.ping, B, dtype, eps, s, nullptr);
  }
  const void* cur = x;
  for (int l = 0; l < L; ++l) {
    BlockWs w = carve_block(ws, B, T, blocks[l]->d, blocks[l]->I, dtype, blocks[l]->w.gnorm != nullptr);
    void* dst = (l == L - 1) ? y : ((l % 2 == 0) ? w.ping : w.pong);
    mmf_status r = block_forward_impl(blocks[l], mmf_state_layer(st, l), cur, dst, B, T, dtype, eps, w, s);
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
