// MLGRU gates + gated linear recurrence over a sequence.
//
// "MatMul-free language models" (DataCamp blog), section "Core components:
// MLGRU and GLU": the MLGRU walks the sequence token by token and updates its
// hidden state with element-wise gates valued in [0,1]; the hysenlabs review,
// section "HGRN attention": forget/candidate paths and a recurrence that only
// sees the current token and the previous state. Per channel:
//   f = sigmoid(f~), c = SiLU(c~), g = sigmoid(g~)
//   h_t = f h_{t-1} + (1 - f) c,   o'_t = g h_t
// The gates live only in registers: the kernel reads the three pre-activation
// rows and writes o' and the final state, nothing else.
#include "kernels.cuh"

namespace mmf {

namespace {

// One thread per (sequence, channel); the loop over tokens is unrolled so the
// loads of later tokens are issued before the recurrence reaches them.
template <typename T>
__global__ void __launch_bounds__(128) mlgru_scan_simple_kernel(const T* __restrict__ pre, int B, int T_, int d,
                                                                float* __restrict__ h, T* __restrict__ o) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * d) return;
  const int b = idx / d, ch = idx % d;
  float hv = h[idx];
  const T* p = pre + (size_t)b * T_ * 3 * d + ch;
  T* op = o + (size_t)b * T_ * d + ch;
#pragma unroll 8
  for (int t = 0; t < T_; ++t) {
    const size_t base = (size_t)t * 3 * d;
    const float f = sigmoidf_(to_f32(p[base]));
    const float c = siluf_(to_f32(p[base + d]));
    const float g = sigmoidf_(to_f32(p[base + 2 * d]));
    hv = f * hv + (1.0f - f) * c;
    op[(size_t)t * d] = from_f32<T>(g * hv);
  }
  h[idx] = hv;
}

}  // namespace

cudaError_t launch_mlgru_scan(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, void* o,
                              cudaStream_t stream) {
  if (B == 0 || T == 0) return cudaSuccess;
  const int n = B * d;
  const int blocks = ceil_div(n, 128);
  if (dt == MMF_BF16)
    mlgru_scan_simple_kernel<bf16><<<blocks, 128, 0, stream>>>(static_cast<const bf16*>(pre), B, T, d, h,
                                                                 static_cast<bf16*>(o));
  else
    mlgru_scan_simple_kernel<float><<<blocks, 128, 0, stream>>>(static_cast<const float*>(pre), B, T, d, h,
                                                                  static_cast<float*>(o));
  return cudaGetLastError();
}

}  // namespace mmf
