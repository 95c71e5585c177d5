// Absmean ternarisation and 2-bit packing of latent weights.
//
// "MatMul-free language models" (DataCamp blog), section "Replacing MatMul
// with ternary operations": the weight matrix is scaled by the mean absolute
// value of its elements and every element is rounded to the nearest of -1, 0, 1.
//
// Two launches, both deterministic for a given (N, K):
//   1. absmean_partial: kPartials CTAs, each sums |W| in fp64 over a fixed
//      grid-stride subset and reduces it in a fixed tree order.
//   2. ternarize_pack: every CTA re-reduces the partials in the same fixed
//      order (so all CTAs see the same gamma), then writes packed words:
//      gamma = (float)(S / (N*K)),  w = clamp(rint(W / (gamma + 1e-5f)), -1, 1),
//      stored value w + 1 at bits 8*b + 2*i of word j for column 16j + 4i + b.
#include "kernels.cuh"

namespace mmf {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ double block_sum_f64(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0) {
    for (int w = 0; w < kThreads / 32; ++w) t += red[w];
    red[0] = t;
  }
  __syncthreads();
  t = red[0];
  __syncthreads();
  return t;
}

__global__ void __launch_bounds__(kThreads) absmean_partial_kernel(const float4* __restrict__ W4, size_t n4,
                                                                   double* __restrict__ partials) {
  __shared__ double red[kThreads / 32];
  double acc = 0.0;
  for (size_t i = (size_t)blockIdx.x * kThreads + threadIdx.x; i < n4; i += (size_t)gridDim.x * kThreads) {
    float4 v = W4[i];
    acc += (double)fabsf(v.x) + (double)fabsf(v.y) + (double)fabsf(v.z) + (double)fabsf(v.w);
  }
  double s = block_sum_f64(acc, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = s;
}

__global__ void __launch_bounds__(kThreads) ternarize_pack_kernel(const float* __restrict__ W, int N, int K,
                                                                  const double* __restrict__ partials, int nparts,
                                                                  float* __restrict__ gamma_out,
                                                                  uint32_t* __restrict__ packed) {
  __shared__ double red[kThreads / 32];
  double v = 0.0;
  for (int i = threadIdx.x; i < nparts; i += kThreads) v += partials[i];
  const double S = block_sum_f64(v, red);
  const float gamma = (float)(S / ((double)N * (double)K));
  if (blockIdx.x == 0 && threadIdx.x == 0) *gamma_out = gamma;
  const float denom = __fadd_rn(gamma, 1e-5f);

  const int wpr = K / 16;                       // words per row
  const size_t nwords = (size_t)N * wpr;
  for (size_t w = (size_t)blockIdx.x * kThreads + threadIdx.x; w < nwords; w += (size_t)gridDim.x * kThreads) {
    const size_t n = w / wpr, j = w % wpr;
    const float4* src = reinterpret_cast<const float4*>(W + n * (size_t)K + j * 16);
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {              // columns 4i .. 4i+3 of this word
      float4 q = src[i];
      float e[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        float t = rintf(__fdiv_rn(e[b], denom));
        int code = (int)fminf(fmaxf(t, -1.0f), 1.0f) + 1;   // 0, 1, 2
        word |= (uint32_t)code << (8 * b + 2 * i);
      }
    }
    packed[w] = word;
  }
}

// One thread per packed word: the 16 stored codes (w + 1) of columns
// 16j .. 16j+15 as 16 bytes, in column order.
__global__ void __launch_bounds__(kThreads) unpack_codes_kernel(const uint32_t* __restrict__ packed, size_t nwords,
                                                                uint4* __restrict__ out) {
  for (size_t w = (size_t)blockIdx.x * kThreads + threadIdx.x; w < nwords; w += (size_t)gridDim.x * kThreads) {
    const uint32_t v = packed[w];
    out[w] = make_uint4(v & 0x03030303u, (v >> 2) & 0x03030303u, (v >> 4) & 0x03030303u, (v >> 6) & 0x03030303u);
  }
}

}  // namespace

cudaError_t launch_unpack_codes(const uint32_t* packed, int N, int K, uint8_t* out, cudaStream_t stream) {
  const size_t nwords = (size_t)N * (K / 16);
  if (nwords == 0) return cudaSuccess;
  const int blocks = (int)std::min<size_t>((nwords + kThreads - 1) / kThreads, (size_t)148 * 16);
  unpack_codes_kernel<<<blocks, kThreads, 0, stream>>>(packed, nwords, reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

size_t quantize_weights_ws_bytes() { return sizeof(double) * kQuantPartials; }

cudaError_t launch_quantize_weights(const float* W, int N, int K, uint32_t* packed, float* gamma, void* ws,
                                    cudaStream_t stream) {
  double* partials = static_cast<double*>(ws);
  const size_t n4 = (size_t)N * K / 4;
  absmean_partial_kernel<<<kQuantPartials, kThreads, 0, stream>>>(reinterpret_cast<const float4*>(W), n4, partials);
  const size_t nwords = (size_t)N * (K / 16);
  int blocks = (int)std::min<size_t>((nwords + kThreads - 1) / kThreads, (size_t)148 * 8);
  if (blocks < 1) blocks = 1;
  ternarize_pack_kernel<<<blocks, kThreads, 0, stream>>>(W, N, K, partials, kQuantPartials, gamma, packed);
  return cudaGetLastError();
}

}  // namespace mmf
