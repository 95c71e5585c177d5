// The two ends of the model around the block stack: the token embedding
// lookup and the greedy next-token choice over the LM head's logits (the head
// itself is a BitLinear d -> V and runs through the contraction kernels).
//
// The hysenlabs review, section "Install and model initialisation": the
// default configuration has an embedding of 32000 entries at hidden size 2048;
// section "FusedBitLinear": every linear projection of the model is a
// FusedBitLinear, the head included. Section "Official generation example"
// samples the next token; the on-device loop here is greedy: the index of the
// largest stored logit, the lowest index on ties.
//
// Both kernels are HBM-bound row streams: the lookup copies M rows of d
// elements with 16-byte vectors (one warp per row), the argmax reads each
// logit row once (one CTA per row).
#include "kernels.cuh"

namespace mmf {

namespace {

constexpr int kEmbedWarps = 8;

// x[m, :] = table[ids[m], :]; an id outside [0, V) writes zeros and records
// status code 8 (reported by mmf_check as an invalid argument).
__global__ void __launch_bounds__(kEmbedWarps * 32)
    embed_kernel(const int32_t* __restrict__ ids, int M, const uint4* __restrict__ table, int V, int vec_per_row,
                 uint4* __restrict__ x, int* status) {
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * kEmbedWarps;
  pdl_trigger();
  pdl_wait();   // ids may be the previous kernel's output (the decode loop's argmax)
  for (int m = blockIdx.x * kEmbedWarps + (threadIdx.x >> 5); m < M; m += nw) {
    const int id = ids[m];
    uint4* dst = x + (size_t)m * vec_per_row;
    if (id < 0 || id >= V) {
      for (int k = lane; k < vec_per_row; k += 32) dst[k] = make_uint4(0u, 0u, 0u, 0u);
      if (lane == 0 && status) atomicExch(status, 8);
      continue;
    }
    const uint4* src = table + (size_t)id * vec_per_row;
    for (int k = lane; k < vec_per_row; k += 32) dst[k] = src[k];
  }
}

// Order of two candidates (value, index): larger value first, a NaN above
// every number, then the lower index.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  const bool vn = v != v, bn = bv != bv;
  if (vn != bn) return vn;
  if (!vn && v != bv) return v > bv;
  return i < bi;
}

__device__ __forceinline__ float elem(const bf16* p, int i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float elem(const float* p, int i) { return p[i]; }

constexpr int kArgThreads = 512;

// ids[m] = argmax_j logits[m, j]; one CTA per row. Each thread scans a strided
// part of the row (16-byte vectors when the row is 16-byte aligned), then a
// shuffle tree and one shared-memory fold pick the winner.
template <typename T>
__global__ void __launch_bounds__(kArgThreads) argmax_kernel(const T* __restrict__ logits, int V, bool vec,
                                                             int32_t* __restrict__ ids) {
  constexpr int E = 16 / sizeof(T);
  __shared__ float sv[kArgThreads / 32];
  __shared__ int si[kArgThreads / 32];
  pdl_trigger();
  pdl_wait();   // the logits are the previous kernel's output
  const T* row = logits + (size_t)blockIdx.x * V;
  float bv = -INFINITY;
  int bi = V;   // no candidate yet: any real element is better (lower index than V on equal value)
  int j0 = 0;
  if (vec) {
    const int nvec = V / E;
    const uint4* rv = reinterpret_cast<const uint4*>(row);
    for (int k = threadIdx.x; k < nvec; k += kArgThreads) {
      const uint4 u = rv[k];
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int q = 0; q < E; ++q) {
        const float v = elem(e, q);
        if (better(v, k * E + q, bv, bi)) {
          bv = v;
          bi = k * E + q;
        }
      }
    }
    j0 = nvec * E;
  }
  for (int j = j0 + threadIdx.x; j < V; j += kArgThreads) {
    const float v = elem(row, j);
    if (better(v, j, bv, bi)) {
      bv = v;
      bi = j;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
    if (better(ov, oi, bv, bi)) {
      bv = ov;
      bi = oi;
    }
  }
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    sv[warp] = bv;
    si[warp] = bi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kArgThreads / 32; ++w)
      if (better(sv[w], si[w], bv, bi)) {
        bv = sv[w];
        bi = si[w];
      }
    ids[blockIdx.x] = bi;
  }
}

}  // namespace

cudaError_t launch_embed(const int32_t* ids, int M, const void* table, int V, int d, mmf_dtype dt, void* x,
                         int* status, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const int vec_per_row = d * (dt == MMF_BF16 ? 2 : 4) / 16;
  const int grid = std::max(1, std::min(ceil_div(M, kEmbedWarps), num_sms() * 8));
  return launch_pdl(embed_kernel, dim3(grid), dim3(kEmbedWarps * 32), 0, stream, ids, M,
                    static_cast<const uint4*>(table), V, vec_per_row, static_cast<uint4*>(x), status);
}

cudaError_t launch_argmax(const void* logits, mmf_dtype dt, int M, int V, int32_t* ids, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const size_t es = dt == MMF_BF16 ? 2 : 4;
  const bool vec = ((uintptr_t)logits % 16 == 0) && (V * es) % 16 == 0;
  if (dt == MMF_BF16)
    return launch_pdl(argmax_kernel<bf16>, dim3(M), dim3(kArgThreads), 0, stream, static_cast<const bf16*>(logits),
                      V, vec, ids);
  return launch_pdl(argmax_kernel<float>, dim3(M), dim3(kArgThreads), 0, stream, static_cast<const float*>(logits),
                    V, vec, ids);
}

}  // namespace mmf
