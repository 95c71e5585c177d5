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

// One warp per token row, the row held in registers as raw 16-byte vectors
// (8 elements each): lane l owns vectors j*32 + l, j < VMAX, so every load and
// every code store of the warp is one contiguous span. Same fp32 steps as the
// CTA-per-row kernel; reductions are warp shuffles only.
template <typename T>
struct Vec16;
template <>
struct Vec16<bf16> {
  using raw = uint4;   // 8 bf16
  static constexpr int regs = 1;
};
template <>
struct Vec16<float> {
  using raw = uint4;   // 4 floats; two raws per 8 elements
  static constexpr int regs = 2;
};

__device__ __forceinline__ void unpack8(const uint4 (&r)[1], float (&v)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r[0]);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void unpack8(const uint4 (&r)[2], float (&v)[8]) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    v[4 * i + 0] = __uint_as_float(r[i].x);
    v[4 * i + 1] = __uint_as_float(r[i].y);
    v[4 * i + 2] = __uint_as_float(r[i].z);
    v[4 * i + 3] = __uint_as_float(r[i].w);
  }
}

// fp32 bit pattern -> the same value as an fp64, built with integer operations
// (the conversion instruction issues at a fraction of the ALU rate). Exact for
// every normal value. Zero and subnormals come out as magnitudes below 2^-126
// instead; their squares stay below 2^-252 and can move a row's sum only when
// every element of the row is that small, and then the fp32 mean square
// underflows to 0 either way.
__device__ __forceinline__ double f32bits_to_f64(uint32_t u) {
  const uint32_t a = u & 0x7fffffffu;          // the sign does not matter for a square
  return __hiloint2double((int)((a >> 3) + 0x38000000u), (int)(a << 29));
}

// Sum of squares of the 8 elements of one raw vector, accumulated in fp64.
__device__ __forceinline__ void sumsq8(const uint4 (&r)[1], double& ss) {
  const uint32_t w[4] = {r[0].x, r[0].y, r[0].z, r[0].w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const double a = f32bits_to_f64(w[i] << 16), b = f32bits_to_f64(w[i] & 0xffff0000u);
    ss = fma(a, a, ss);
    ss = fma(b, b, ss);
  }
}
__device__ __forceinline__ void sumsq8(const uint4 (&r)[2], double& ss) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t w[4] = {r[i].x, r[i].y, r[i].z, r[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const double a = f32bits_to_f64(w[k]);
      ss = fma(a, a, ss);
    }
  }
}

// rint(t) for |t| < 2^22 by adding 1.5 * 2^23: the sum's unit in the last
// place is 1, so the fp32 add rounds t half-to-even to an integer, and the
// sum's bit pattern is 0x4B400000 + rint(t) with rint(t) in two's complement
// in the low bits. Returns that bit pattern; its low byte is the int8 code.
__device__ __forceinline__ uint32_t rint_bits(float t) { return __float_as_uint(__fadd_rn(t, 12582912.0f)); }

// Low bytes of four rint_bits() patterns -> one word, bytes in order a, b, c, d.
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

template <typename T, int VMAX>
__device__ __forceinline__ void load_row(const T* __restrict__ xr, int nvec, int lane, uint4 (&raw)[VMAX][Vec16<T>::regs]) {
  constexpr int R = Vec16<T>::regs;
#pragma unroll
  for (int j = 0; j < VMAX; ++j) {
    const int vi = j * 32 + lane;
#pragma unroll
    for (int r = 0; r < R; ++r)
      raw[j][r] = vi < nvec ? __ldg(reinterpret_cast<const uint4*>(xr + (size_t)vi * 8) + r) : make_uint4(0, 0, 0, 0);
  }
}

// Persistent: each warp walks rows warp_id, warp_id + nwarps, ... and issues
// the loads of its next row before reducing the current one, so the row's
// HBM latency overlaps the previous row's arithmetic.
template <typename T, int VMAX>
__global__ void __launch_bounds__(256) rmsnorm_quant_warp_kernel(const T* __restrict__ x, int M, int K,
                                                                 const float* __restrict__ gain, float eps,
                                                                 int8_t* __restrict__ q, float* __restrict__ scale,
                                                                 int32_t* __restrict__ qsum) {
  constexpr int R = Vec16<T>::regs;
  constexpr bool kKeep = VMAX <= 8;   // keep x^ in registers between the max and the codes
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * 8;
  int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  pdl_trigger();
  pdl_wait();
  if (row >= M) return;
  const int nvec = K / 8;
  uint4 raw[VMAX][R], nxt[VMAX][R];
  load_row<T, VMAX>(x + (size_t)row * K, nvec, lane, raw);
  for (; row < M; row += nwarps) {
    if (row + nwarps < M) load_row<T, VMAX>(x + (size_t)(row + nwarps) * K, nvec, lane, nxt);
    double ss = 0.0;
#pragma unroll
    for (int j = 0; j < VMAX; ++j) sumsq8(raw[j], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float ms = (float)(ss / (double)K);
    const float rinv = __frcp_rn(__fsqrt_rn(__fadd_rn(ms, eps)));

    float xh[kKeep ? VMAX : 1][8];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < VMAX; ++j) {
      const int vi = j * 32 + lane;
      float v[8];
      unpack8(raw[j], v);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float h = __fmul_rn(v[i], rinv);
        if (gain != nullptr && vi < nvec) h = __fmul_rn(h, __ldg(gain + vi * 8 + i));
        amax = fmaxf(amax, fabsf(h));
        if constexpr (kKeep) xh[j][i] = h;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));

    int isum = 0;
    int8_t* qr = q + (size_t)row * K;
#pragma unroll
    for (int j = 0; j < VMAX; ++j) {
      const int vi = j * 32 + lane;
      if (vi >= nvec) break;
      float h[8];
      if constexpr (kKeep) {
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = xh[j][i];
      } else {
        float v[8];
        unpack8(raw[j], v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          h[i] = __fmul_rn(v[i], rinv);
          if (gain != nullptr) h[i] = __fmul_rn(h[i], __ldg(gain + vi * 8 + i));
        }
      }
      // |x^ * s| <= 127 (to within rounding) by the choice of s, so the codes
      // need no clamp and never reach -128
      uint32_t c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = rint_bits(__fmul_rn(h[i], s));
      const uint32_t w0 = pack_low_bytes(c[0], c[1], c[2], c[3]);
      const uint32_t w1 = pack_low_bytes(c[4], c[5], c[6], c[7]);
      isum = __dp4a((int)w0, 0x01010101, isum);
      isum = __dp4a((int)w1, 0x01010101, isum);
      *reinterpret_cast<uint2*>(qr + (size_t)vi * 8) = make_uint2(w0, w1);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) isum += __shfl_xor_sync(0xffffffffu, isum, o);
    if (lane == 0) {
      scale[row] = s;
      qsum[row] = isum;
    }
#pragma unroll
    for (int j = 0; j < VMAX; ++j)
#pragma unroll
      for (int r = 0; r < R; ++r) raw[j][r] = nxt[j][r];
  }
}

template <typename T, int VMAX>
void launch_warp(const void* x, int M, int K, const float* gain, float eps, int8_t* q, float* scale, int32_t* qsum,
                 cudaStream_t stream) {
  auto kern = rmsnorm_quant_warp_kernel<T, VMAX>;
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0);
  const int grid = std::max(1, std::min(ceil_div(M, 8), num_sms() * std::max(per_sm, 1)));
  launch_pdl(kern, dim3(grid), dim3(256), 0, stream, static_cast<const T*>(x), M, K, gain, eps, q, scale, qsum);
}

}  // namespace

cudaError_t launch_rmsnorm_quant(const void* x, mmf_dtype dt, int M, int K, const float* gain, float eps,
                                 int8_t* q, float* scale, int32_t* qsum, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  // warp-per-row kernels while two rows fit in registers (K / 256 vectors per lane)
  const int vpl = ceil_div(K / 8, 32);
  if (dt == MMF_BF16 && vpl <= 12) {
    if (vpl <= 4) launch_warp<bf16, 4>(x, M, K, gain, eps, q, scale, qsum, stream);
    else if (vpl <= 8) launch_warp<bf16, 8>(x, M, K, gain, eps, q, scale, qsum, stream);
    else launch_warp<bf16, 12>(x, M, K, gain, eps, q, scale, qsum, stream);
    return cudaGetLastError();
  }
  if (dt == MMF_F32 && vpl <= 4) {
    launch_warp<float, 4>(x, M, K, gain, eps, q, scale, qsum, stream);
    return cudaGetLastError();
  }
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
