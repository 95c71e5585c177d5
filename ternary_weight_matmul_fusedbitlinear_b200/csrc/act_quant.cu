// Fused RMSNorm + per-token absmax int8 quantisation (the BitLinear prologue).
//
// "MatMul-free language models" (DataCamp blog), overview figure panel
// "RMS Norm": activations are normalised before they are quantised; the
// hysenlabs review, section "FusedBitLinear": RMSNorm on the input, then the
// fused quantise-and-accumulate kernel. Per token row x[0..K):
//   ms  = (float)(sum x^2 in fp64 / K)
//   r   = sqrt(ms + eps);  rinv = 1 / r                 (IEEE fp32)
//   x^  = (x * rinv) * gain                              (IEEE fp32 products)
//   s   = 127 / max(max|x^|, 1e-5)
//   q   = clamp(rint(x^ * s), -128, 127),  qsum = sum q  (int32)
// Every fp32 step is a correctly rounded single operation, so the codes do not
// depend on how the kernel is laid out; only the fp64 sum's order could, and
// it is fixed here (per-thread strided order, xor-shuffle tree, warps in order).
#include "kernels.cuh"

namespace mmf {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <typename T>
__global__ void __launch_bounds__(kThreads) rmsnorm_quant_kernel(const T* __restrict__ x, int K,
                                                                 const float* __restrict__ gain, float eps,
                                                                 int8_t* __restrict__ q, float* __restrict__ scale,
                                                                 int32_t* __restrict__ qsum) {
  extern __shared__ float xs[];  // K floats
  __shared__ double red_d[kWarps];
  __shared__ float red_f[kWarps];
  __shared__ int red_i[kWarps];
  const int row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* xr = x + (size_t)row * K;

  // pass 1: load (8 per thread per step), keep in shared memory, sum of squares in fp64
  double ss = 0.0;
  for (int k = threadIdx.x * 8; k < K; k += kThreads * 8) {
    float v[8];
    load8(xr + k, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      xs[k + i] = v[i];
      ss += (double)v[i] * (double)v[i];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red_d[warp] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kWarps; ++w) t += red_d[w];
    red_d[0] = t;
  }
  __syncthreads();
  const float ms = (float)(red_d[0] / (double)K);
  const float r = __fsqrt_rn(__fadd_rn(ms, eps));
  const float rinv = __frcp_rn(r);

  // pass 2: x^ and its absolute maximum
  float amax = 0.0f;
  for (int k = threadIdx.x; k < K; k += kThreads) {
    float v = __fmul_rn(xs[k], rinv);
    if (gain != nullptr) v = __fmul_rn(v, gain[k]);
    xs[k] = v;
    amax = fmaxf(amax, fabsf(v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) red_f[warp] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.0f;
    for (int w = 0; w < kWarps; ++w) t = fmaxf(t, red_f[w]);
    red_f[0] = t;
  }
  __syncthreads();
  const float s = __fdiv_rn(127.0f, fmaxf(red_f[0], 1e-5f));

  // pass 3: codes, 4 per thread per step (one 32-bit store)
  int isum = 0;
  int8_t* qr = q + (size_t)row * K;
  for (int k = threadIdx.x * 4; k < K; k += kThreads * 4) {
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int c = __float2int_rn(__fmul_rn(xs[k + i], s));
      c = max(-128, min(127, c));
      isum += c;
      packed |= (uint32_t)(c & 0xff) << (8 * i);
    }
    *reinterpret_cast<uint32_t*>(qr + k) = packed;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) isum += __shfl_xor_sync(0xffffffffu, isum, o);
  if (lane == 0) red_i[warp] = isum;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < kWarps; ++w) t += red_i[w];
    scale[row] = s;
    qsum[row] = t;
  }
}

}  // namespace

cudaError_t launch_rmsnorm_quant(const void* x, mmf_dtype dt, int M, int K, const float* gain, float eps,
                                 int8_t* q, float* scale, int32_t* qsum, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * (size_t)K;
  if (dt == MMF_BF16) {
    auto kern = rmsnorm_quant_kernel<bf16>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<M, kThreads, smem, stream>>>(static_cast<const bf16*>(x), K, gain, eps, q, scale, qsum);
  } else {
    auto kern = rmsnorm_quant_kernel<float>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<M, kThreads, smem, stream>>>(static_cast<const float*>(x), K, gain, eps, q, scale, qsum);
  }
  return cudaGetLastError();
}

}  // namespace mmf
