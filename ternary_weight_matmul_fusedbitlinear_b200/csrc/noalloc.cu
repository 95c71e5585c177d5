// mmf_bitlinear_noalloc: the FusedBitLinear forward for callers that cannot
// allocate device memory and cannot hand the library a workspace.
//
// Who needs it: code that receives only its input and output buffers, such as
// a custom-operator plug-in of another framework or serving engine whose
// interface passes tensors but no scratch, and processes that reserve their
// whole device-memory budget up front, where a cudaMalloc in the middle of a
// request would fail or fragment that budget. mmf_bitlinear wants a
// caller-owned workspace for the int8 activation codes, their scales and
// their row sums; this variant keeps those in one fixed array that is part of
// the library image instead.
//
// The array lives in device memory of every GPU that loads the library and
// stays there until the process exits. All calls share it and it keeps the
// last call's contents; every kernel here overwrites what it later reads, so
// nothing needs clearing. Calls whose work overlaps on the GPU (two streams,
// two threads) race on the array and must be serialised by the caller.
#include <cstdio>
#include <mutex>

#include "kernels.cuh"

namespace mmf {
namespace {

constexpr size_t kNoallocBytes = (size_t)MMF_NOALLOC_SCRATCH_BYTES;

// The scratch itself. In host code this name is only a host-side stand-in for
// the symbol, never a device address: its device address comes from
// cudaGetSymbolAddress below, per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

inline size_t up256(size_t v) { return (v + 255) / 256 * 256; }

// Bytes of scratch needed for M tokens of length K: codes, scales, row sums.
inline size_t need_bytes(int M, int K) { return up256((size_t)M * K) + 2 * up256(sizeof(float) * (size_t)M); }

}  // namespace
}  // namespace mmf

using namespace mmf;

namespace {

mmf_status noalloc_fail(mmf_status st, const char* msg) {
  set_last_error(msg);
  return st;
}

}  // namespace

extern "C" mmf_status mmf_bitlinear_noalloc(const mmf_tlinear* lin, const void* x, mmf_dtype dtype, int32_t M,
                                            void* y, float eps, void* stream) {
  char msg[256];
  if (lin == nullptr || lin->packed == nullptr || lin->gamma == nullptr)
    return noalloc_fail(MMF_ERR_INVALID_ARG, "mmf_bitlinear_noalloc: null layer");
  if (lin->N < 1 || lin->K < 1 || M < 0) return noalloc_fail(MMF_ERR_INVALID_ARG, "mmf_bitlinear_noalloc: bad sizes");
  if (lin->K % 16 != 0) return noalloc_fail(MMF_ERR_UNSUPPORTED_SHAPE, "mmf_bitlinear_noalloc: K % 16 != 0");
  if (dtype != MMF_F32 && dtype != MMF_BF16) return noalloc_fail(MMF_ERR_INVALID_ARG, "mmf_bitlinear_noalloc: dtype");
  if (!(eps > 0.0f)) return noalloc_fail(MMF_ERR_INVALID_ARG, "mmf_bitlinear_noalloc: eps must be > 0");
  if (M == 0) return MMF_OK;
  if (x == nullptr || y == nullptr) return noalloc_fail(MMF_ERR_INVALID_ARG, "mmf_bitlinear_noalloc: null x/y");
  if (((uintptr_t)x | (uintptr_t)y | (uintptr_t)lin->packed) & 15u)
    return noalloc_fail(MMF_ERR_MISALIGNED, "mmf_bitlinear_noalloc: pointer not 16-byte aligned");
  // the same layer checks as mmf_bitlinear: optional vectors must be 16-byte aligned too
  if (((uintptr_t)lin->gain | (uintptr_t)lin->bias | (uintptr_t)lin->codes) & 15u)
    return noalloc_fail(MMF_ERR_MISALIGNED, "mmf_bitlinear_noalloc: gain/bias/codes not 16-byte aligned");
  if (need_bytes(M, lin->K) > kNoallocBytes) {
    snprintf(msg, sizeof(msg),
             "mmf_bitlinear_noalloc: M=%d x K=%d needs %zu bytes of scratch, more than the fixed %zu-byte "
             "array; split the tokens or use mmf_bitlinear with a workspace",
             M, lin->K, need_bytes(M, lin->K), kNoallocBytes);
    return noalloc_fail(MMF_ERR_UNSUPPORTED_SHAPE, msg);
  }

  // Set-up, once per device, with that device current: the array's device address.
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return noalloc_fail(MMF_ERR_CUDA, "mmf_bitlinear_noalloc: cudaGetDevice failed");
  void* base = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || p == nullptr) {
        snprintf(msg, sizeof(msg), "mmf_bitlinear_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
        return noalloc_fail(MMF_ERR_CUDA, msg);
      }
      g_scratch_addr[dev] = p;
    }
    base = g_scratch_addr[dev];
  }

  char* cur = static_cast<char*>(base);
  int8_t* q = reinterpret_cast<int8_t*>(cur);
  cur += up256((size_t)M * lin->K);
  float* s = reinterpret_cast<float*>(cur);
  cur += up256(sizeof(float) * (size_t)M);
  int32_t* qsum = reinterpret_cast<int32_t*>(cur);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // no status word here (obtaining it may allocate): a timed-out wait in the
  // quantiser leaves its rows unwritten without a recorded code
  e = launch_rmsnorm_quant(x, dtype, M, lin->K, lin->gain, eps, q, s, qsum, nullptr, st);
  if (e == cudaSuccess) {
    TGemmArgs a{};
    for (int i = 0; i < 3; ++i) {
      a.w[i] = lin->packed;
      a.gamma[i] = lin->gamma;
      a.bias[i] = lin->bias;
    }
    a.nseg = 1;
    a.N = lin->N;
    a.K = lin->K;
    a.q = q;
    a.s = s;
    a.qsum = qsum;
    a.M = M;
    a.out = y;
    a.ldo = lin->N;
    e = launch_tgemm_mma(a, Epi::kStore, dtype, st);
  }
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "mmf_bitlinear_noalloc: launch failed: %s", cudaGetErrorString(e));
    return noalloc_fail(MMF_ERR_CUDA, msg);
  }
  return MMF_OK;
}
