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
#include "tma.cuh"
#include "quant_row.cuh"

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

// ---------------------------------------------------------------- staged warp-per-row kernel
// One warp per token row. Each warp keeps a ring of `slots` row buffers in
// shared memory and fills them with 1-D bulk copies (cp.async.bulk, one per
// row), so the next rows stream in while the current one is reduced; the row
// itself is read from shared memory by quant_row(), never from HBM again.

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Bounded wait on a row buffer (all lanes); false after the time limit, with
// status code 1 recorded when a status word is given.
__device__ __forceinline__ bool slot_wait(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) {
      if (status && (threadIdx.x & 31) == 0) atomicExch(status, 1);
      return false;
    }
  }
  return true;
}

template <typename T, bool GAIN>
__global__ void __launch_bounds__(256) rmsnorm_quant_staged_kernel(const T* __restrict__ x, int M, int K,
                                                                   const float* __restrict__ gain, float eps,
                                                                   int8_t* __restrict__ q, float* __restrict__ scale,
                                                                   int32_t* __restrict__ qsum, int slots,
                                                                   int stride, int* status, uint4* fill,
                                                                   size_t fill16) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = base + (size_t)warp * slots * stride;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + (size_t)warps * slots * stride) + warp * slots;
  const int nwarps = gridDim.x * warps;
  const int row0 = blockIdx.x * warps + warp;
  const uint32_t row_bytes = (uint32_t)K * sizeof(T);
  const int nvec = (int)(row_bytes / 16);

  if (lane == 0) {
    for (int s = 0; s < slots; ++s) mbar_init(&bars[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  pdl_trigger();
  pdl_wait();   // x is the previous kernel's output
  // side work for a later kernel: fill `fill16` 16-byte units with all-ones bytes
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < fill16; i += (size_t)gridDim.x * blockDim.x)
    fill[i] = make_uint4(~0u, ~0u, ~0u, ~0u);
  if (lane == 0) {
    for (int s = 0; s < slots; ++s) {
      const int r = row0 + s * nwarps;
      if (r >= M) break;
      mbar_arrive_expect_tx(&bars[s], row_bytes);
      bulk_load(ring + (size_t)s * stride, x + (size_t)r * K, row_bytes, &bars[s]);
    }
  }

  int k = 0;
  for (int row = row0; row < M; row += nwarps, ++k) {
    const int s = k % slots;
    if (!slot_wait(&bars[s], (uint32_t)(k / slots) & 1u, status)) {
      // give up on this warp's rows; let the copies in flight land (bounded)
      if (lane == 0)
        for (int i = 1; i < slots; ++i) {
          const int si = (k + i) % slots;
          if (row + i * nwarps < M) slot_wait(&bars[si], (uint32_t)((k + i) / slots) & 1u, nullptr);
        }
      return;
    }
    const uint4* v = reinterpret_cast<const uint4*>(ring + (size_t)s * stride);
    const RowCode rc = quant_row<T, GAIN, false>(v, nvec, K, gain, eps, q + (size_t)row * K, lane);
    if (lane == 0) {
      scale[row] = rc.scale;
      qsum[row] = rc.qsum;
    }

    // refill this buffer with the row `slots` rows ahead
    __syncwarp();
    if (lane == 0) {
      const int nr = row + slots * nwarps;
      if (nr < M) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[s], row_bytes);
        bulk_load(ring + (size_t)s * stride, x + (size_t)nr * K, row_bytes, &bars[s]);
      }
    }
  }
}

// Geometry of the staged kernel for one row length; false when a row does not fit.
struct StagedGeom {
  int warps, slots, stride;
  size_t smem;
};
bool staged_geometry(int K, int esize, StagedGeom& g) {
  g.stride = (K * esize + 127) / 128 * 128;
  constexpr int kBudget = 200 * 1024;   // shared memory per CTA
  g.warps = 2 * 8 * g.stride <= kBudget ? 8 : 4;
  if (2 * g.warps * g.stride > kBudget) return false;
  g.slots = std::max(2, std::min(4, (96 * 1024) / (g.warps * g.stride)));
  g.smem = (size_t)g.warps * g.slots * g.stride + sizeof(uint64_t) * g.warps * g.slots + 128;
  return true;
}

template <typename T, bool GAIN>
cudaError_t launch_staged(const StagedGeom& g, const void* x, int M, int K, const float* gain, float eps, int8_t* q,
                          float* scale, int32_t* qsum, int* status, void* fill, size_t fill_bytes, cudaStream_t stream) {
  auto kern = rmsnorm_quant_staged_kernel<T, GAIN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.smem);
  if (e != cudaSuccess) return e;
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, g.warps * 32, g.smem);
  const int grid = std::max(1, std::min(ceil_div(M, g.warps), num_sms() * std::max(per_sm, 1)));
  return launch_pdl(kern, dim3(grid), dim3(g.warps * 32), g.smem, stream, static_cast<const T*>(x), M, K, gain, eps,
                    q, scale, qsum, g.slots, g.stride, status, static_cast<uint4*>(fill), fill_bytes / 16);
}

}  // namespace

cudaError_t launch_rmsnorm_quant(const void* x, mmf_dtype dt, int M, int K, const float* gain, float eps,
                                 int8_t* q, float* scale, int32_t* qsum, int* status, cudaStream_t stream, void* fill,
                                 size_t fill_bytes) {
  if (M == 0) return fill_bytes ? cudaMemsetAsync(fill, 0xff, fill_bytes, stream) : cudaSuccess;
  StagedGeom g;
  if (staged_geometry(K, dt == MMF_BF16 ? 2 : 4, g) && fill_bytes % 16 == 0) {
    if (dt == MMF_BF16)
      return gain ? launch_staged<bf16, true>(g, x, M, K, gain, eps, q, scale, qsum, status, fill, fill_bytes, stream)
                  : launch_staged<bf16, false>(g, x, M, K, gain, eps, q, scale, qsum, status, fill, fill_bytes, stream);
    return gain ? launch_staged<float, true>(g, x, M, K, gain, eps, q, scale, qsum, status, fill, fill_bytes, stream)
                : launch_staged<float, false>(g, x, M, K, gain, eps, q, scale, qsum, status, fill, fill_bytes, stream);
  }
  if (fill_bytes) {
    const cudaError_t e = cudaMemsetAsync(fill, 0xff, fill_bytes, stream);
    if (e != cudaSuccess) return e;
  }
  // rows too long for the staged ring: one CTA per row
  const size_t smem = sizeof(float) * (size_t)K;
  if (dt == MMF_BF16) {
    auto kern = rmsnorm_quant_kernel<bf16>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<M, kThreads, smem, stream>>>(static_cast<const bf16*>(x), K, gain, eps, q, scale, qsum);
  } else {
    auto kern = rmsnorm_quant_kernel<float>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<M, kThreads, smem, stream>>>(static_cast<const float*>(x), K, gain, eps, q, scale, qsum);
  }
  return cudaGetLastError();
}

}  // namespace mmf
