// One token row of the fused RMSNorm + absmax int8 quantisation, computed by
// one warp (sm_100a). Shared by the standalone quantiser and by the decode
// contraction, which quantises its few token rows itself.
//
// "MatMul-free language models" (DataCamp blog), overview figure panel
// "RMS Norm", and the hysenlabs review, section "FusedBitLinear": RMSNorm on
// the input, then per-token absmax quantisation to int8. Per row x[0..K):
//   ms  = (float)(sum x^2 in fp64 / K)
//   rinv = 1 / sqrt(ms + eps)                        (IEEE fp32)
//   x^  = (x * rinv) * gain                          (IEEE fp32 products)
//   s   = 127 / max(max|x^|, 1e-5)
//   q   = rint(x^ * s) (|x^ s| <= 127 up to rounding, so no clamp is needed
//         and -128 never occurs),  qsum = sum q      (int32)
// Every fp32 step is a correctly rounded single operation, so the codes do not
// depend on the kernel's layout; the fp64 sum's order is fixed (lane l sums
// vectors l, l+32, ... in order, then an xor-shuffle tree).
// Pass 1 sums the squares and takes max|x|. Without a gain vector that already
// fixes the scale: rounding is monotone, so fl(max|x| * rinv) =
// max fl(|x| * rinv) = max|x^|. With a gain vector a second pass takes
// max|(x * rinv) * gain|. The last pass writes the codes.
#pragma once

#include "common.cuh"

namespace mmf {

// fp32 bit pattern (sign cleared) -> the same value as an fp64, built with
// integer operations (the conversion instruction issues at a fraction of the
// ALU rate). Exact for every normal value. Zero and subnormals come out as
// magnitudes below 2^-126 instead; their squares stay below 2^-252 and can
// move a row's sum only when every element of the row is that small, and then
// the fp32 mean square underflows to 0 either way.
__device__ __forceinline__ double magbits_to_f64(uint32_t a) {
  return __hiloint2double((int)((a >> 3) + 0x38000000u), (int)(a << 29));
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

// Per element type: E elements per 16-byte vector, their fp32 magnitude bits
// and values.
template <typename T>
struct Vec;
template <>
struct Vec<bf16> {
  static constexpr int E = 8;
  __device__ __forceinline__ static uint32_t mag(const uint4& r, int i) {
    const uint32_t w = (&r.x)[i >> 1];
    return (i & 1) ? (w & 0x7fff0000u) : ((w << 16) & 0x7fffffffu);
  }
  __device__ __forceinline__ static float val(const uint4& r, int i) {
    const uint32_t w = (&r.x)[i >> 1];
    return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
  }
  __device__ __forceinline__ static void store_codes(int8_t* p, const uint32_t (&c)[8], int& isum) {
    const uint32_t w0 = pack_low_bytes(c[0], c[1], c[2], c[3]);
    const uint32_t w1 = pack_low_bytes(c[4], c[5], c[6], c[7]);
    isum = __dp4a((int)w0, 0x01010101, isum);
    isum = __dp4a((int)w1, 0x01010101, isum);
    *reinterpret_cast<uint2*>(p) = make_uint2(w0, w1);
  }
};
template <>
struct Vec<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static uint32_t mag(const uint4& r, int i) { return (&r.x)[i] & 0x7fffffffu; }
  __device__ __forceinline__ static float val(const uint4& r, int i) { return __uint_as_float((&r.x)[i]); }
  __device__ __forceinline__ static void store_codes(int8_t* p, const uint32_t (&c)[4], int& isum) {
    const uint32_t w0 = pack_low_bytes(c[0], c[1], c[2], c[3]);
    isum = __dp4a((int)w0, 0x01010101, isum);
    *reinterpret_cast<uint32_t*>(p) = w0;
  }
};

struct RowCode {
  float scale;
  int qsum;
};

// Warp-collective: all 32 lanes call it with the same row. `v` points at the
// row as nvec 16-byte vectors (K elements), in global memory when GLOBAL
// (read through the read-only path) or in shared memory; codes go to qr
// (16-byte aligned, global or shared). With INPLACE, qr is the row itself: the
// codes of vector vi overwrite bytes [E vi, E vi + E), which hold vectors read
// in the same or an earlier step of the last pass, and a compiler barrier
// keeps each step's accesses in program order. Returns the scale and the code
// sum on every lane.
template <typename T, bool GAIN, bool GLOBAL, bool INPLACE = false>
__device__ __forceinline__ RowCode quant_row(const uint4* v, int nvec, int K, const float* __restrict__ gain,
                                             float eps, int8_t* qr, int lane) {
  using V = Vec<T>;
  constexpr int E = V::E;
  auto ld = [&](int vi) -> uint4 {
    if constexpr (GLOBAL) return __ldg(v + vi);
    else return v[vi];
  };
  // pass 1: sum of squares (fp64) and max |x|
  double ss = 0.0;
  uint32_t am = 0;
#pragma unroll 4
  for (int vi = lane; vi < nvec; vi += 32) {
    const uint4 r = ld(vi);
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const uint32_t a = V::mag(r, i);
      am = max(am, a);
      const double xd = magbits_to_f64(a);
      ss = fma(xd, xd, ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float ms = (float)(ss / (double)K);
  const float rinv = __frcp_rn(__fsqrt_rn(__fadd_rn(ms, eps)));

  float amax;
  if constexpr (GAIN) {   // pass 2: max |(x * rinv) * gain|
    uint32_t hm = 0;
#pragma unroll 4
    for (int vi = lane; vi < nvec; vi += 32) {
      const uint4 r = ld(vi);
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const float hv = __fmul_rn(__fmul_rn(V::val(r, i), rinv), __ldg(gain + vi * E + i));
        hm = max(hm, __float_as_uint(hv) & 0x7fffffffu);
      }
    }
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, hm));
  } else {
    amax = __fmul_rn(__uint_as_float(__reduce_max_sync(0xffffffffu, am)), rinv);
  }
  const float sc = __fdiv_rn(127.0f, fmaxf(amax, 1e-5f));

  // last pass: codes and their sum
  int isum = 0;
#pragma unroll 4
  for (int vi = lane; vi < nvec; vi += 32) {
    const uint4 r = ld(vi);
    uint32_t c[E];
#pragma unroll
    for (int i = 0; i < E; ++i) {
      float hv = __fmul_rn(V::val(r, i), rinv);
      if constexpr (GAIN) hv = __fmul_rn(hv, __ldg(gain + vi * E + i));
      c[i] = rint_bits(__fmul_rn(hv, sc));
    }
    V::store_codes(qr + (size_t)vi * E, c, isum);
    if constexpr (INPLACE) asm volatile("" ::: "memory");
  }
  return RowCode{sc, __reduce_add_sync(0xffffffffu, isum)};
}

}  // namespace mmf

namespace mmf {

// Block-wide form of the same quantisation for a few token rows at once (at
// most MPAD rows; NT threads, NT / MPAD >= 32 threads per row). Thread t works
// on row t / (NT / MPAD) and holds that row's 16-byte vectors lt, lt + tpr, ...
// (lt = t % tpr, tpr = NT / MPAD) in raw[j] for every bit j set in `have`. The
// row's fp64 sum of squares and its max are reduced in a fixed order (lanes by
// an xor-shuffle tree, then the row's warps by a shuffle tree), so every CTA
// that quantises the same rows gets the same scale; every warp of a row folds
// the row's partials itself, so no thread waits for another's fold. The fp32
// steps are those of quant_row. Codes go to codes + m * qpitch (16-byte aligned
// rows) and scale[m] gets the row's scale. The code sums are left as per-warp
// partials in red.i: block_qsum() folds them after the caller's next barrier.
// `red` is shared scratch of NT / 32 entries of each type. Contains
// __syncthreads(): every thread of the block calls it. `fail` (any thread)
// makes every thread return false right after the first barrier, with
// nothing written; the barrier doubles as the caller's vote on giving up.
struct BlockRed {
  double* d;
  uint32_t* u;
  int* i;
};

// Fold a row's kWpr per-warp partials (red[w0 .. w0 + kWpr)) in a fixed tree
// order; every lane gets the result.
template <int kWpr, typename V, typename Op>
__device__ __forceinline__ V fold_row(const V* red, int w0, int lane, V zero, Op op) {
  V v = lane < kWpr ? red[w0 + lane] : zero;
#pragma unroll
  for (int o = kWpr / 2; o > 0; o >>= 1) {
    const V other = __shfl_down_sync(0xffffffffu, v, o);
    if (lane < o) v = op(v, other);
  }
  return __shfl_sync(0xffffffffu, v, 0);
}

template <typename T, int MPAD, int NT, int VMAX>
__device__ __forceinline__ bool block_quant(const uint4 (&raw)[VMAX], uint32_t have, int M, int K,
                                            const float* __restrict__ gain, float eps, int8_t* codes, int qpitch,
                                            float* scale, const BlockRed& red, bool fail = false) {
  using V = Vec<T>;
  constexpr int E = V::E;
  constexpr int kTpr = NT / MPAD;
  constexpr int kWpr = kTpr / 32;
  static_assert(kTpr >= 32 && (kWpr & (kWpr - 1)) == 0, "a power-of-two number of warps per row");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m_row = tid / kTpr, lt = tid - m_row * kTpr;
  const int w0 = m_row * kWpr;
  const bool row_ok = m_row < M;
  // A thread's slots are a prefix of 0..VMAX-1 (vector lt + tpr j is in the row
  // for every j below some bound), so the unrolled loops stop at the first
  // empty slot instead of running predicated bodies for all VMAX slots.
  {   // sum of squares (fp64, two chains: even and odd elements) and max |x|
    double s0 = 0.0, s1 = 0.0;
    uint32_t am = 0;
#pragma unroll
    for (int j = 0; j < VMAX; ++j) {
      if (!(have & (1u << j))) break;
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const uint32_t mg = V::mag(raw[j], i);
        am = max(am, mg);
        const double xd = magbits_to_f64(mg);
        if (i & 1) s1 = fma(xd, xd, s1);
        else s0 = fma(xd, xd, s0);
      }
    }
    double ss = s0 + s1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    am = __reduce_max_sync(0xffffffffu, am);
    if (lane == 0) {
      red.d[warp] = ss;
      red.u[warp] = am;
    }
  }
  if (__syncthreads_or(fail)) return false;
  const double tot = fold_row<kWpr>(red.d, w0, lane, 0.0, [](double x, double y) { return x + y; });
  const uint32_t mx = fold_row<kWpr>(red.u, w0, lane, 0u, [](uint32_t x, uint32_t y) { return max(x, y); });
  const float ms = (float)(tot / (double)K);
  const float rinv = __frcp_rn(__fsqrt_rn(__fadd_rn(ms, eps)));
  float sc;
  if (gain == nullptr) {   // rounding is monotone: fl(max|x| * rinv) = max fl(|x| * rinv)
    sc = __fdiv_rn(127.0f, fmaxf(__fmul_rn(__uint_as_float(mx), rinv), 1e-5f));
  } else {   // max |(x * rinv) * gain|
    uint32_t hm = 0;
#pragma unroll
    for (int j = 0; j < VMAX; ++j) {
      if (!(have & (1u << j))) break;
      const int k0 = (lt + kTpr * j) * E;
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const float hv = __fmul_rn(__fmul_rn(V::val(raw[j], i), rinv), __ldg(gain + k0 + i));
        hm = max(hm, __float_as_uint(hv) & 0x7fffffffu);
      }
    }
    hm = __reduce_max_sync(0xffffffffu, hm);
    __syncthreads();   // every warp has read the first partials
    if (lane == 0) red.u[warp] = hm;
    __syncthreads();
    const uint32_t gm = fold_row<kWpr>(red.u, w0, lane, 0u, [](uint32_t x, uint32_t y) { return max(x, y); });
    sc = __fdiv_rn(127.0f, fmaxf(__uint_as_float(gm), 1e-5f));
  }
  if (row_ok && lt == 0) scale[m_row] = sc;
  {   // codes and this warp's part of their sum
    int isum = 0;
#pragma unroll
    for (int j = 0; j < VMAX; ++j) {
      if (!(have & (1u << j))) break;
      const int v = lt + kTpr * j;
      uint32_t c[E];
#pragma unroll
      for (int i = 0; i < E; ++i) {
        float hv = __fmul_rn(V::val(raw[j], i), rinv);
        if (gain != nullptr) hv = __fmul_rn(hv, __ldg(gain + v * E + i));
        c[i] = rint_bits(__fmul_rn(hv, sc));
      }
      V::store_codes(codes + (size_t)m_row * qpitch + v * E, c, isum);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) isum += __shfl_xor_sync(0xffffffffu, isum, o);
    if (lane == 0) red.i[warp] = isum;
  }
  __syncthreads();
  return true;
}

// Code sum of row m from block_quant's per-warp partials (any thread, after block_quant).
template <int MPAD, int NT>
__device__ __forceinline__ int block_qsum(const BlockRed& red, int m) {
  constexpr int kWpr = NT / MPAD / 32;
  int t = 0;
#pragma unroll
  for (int w = 0; w < kWpr; ++w) t += red.i[m * kWpr + w];
  return t;
}

}  // namespace mmf
