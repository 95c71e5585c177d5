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
// rows once and writes o' and the final state, nothing else.
//
// g_norm output gate (the hysenlabs review, same section: g_norm is a
// FusedRMSNormSwishGate). o'_t = h_t / sqrt(mean_n h_t^2 + eps) * w * swish(g~_t)
// needs the whole token row of h, which no CTA holds, so it takes two
// kernels: the scan (GN = true) computes swish(g~) in place of sigmoid(g~),
// writes v_t = swish(g~_t) h_t in fp32 and, per token and channel block, the
// partial sum of h_t^2; gnorm_apply_kernel adds a row's partials and writes
// o' = v * (1 / sqrt(sum / d + eps)) * w in the storage type. Inside a block
// the o projection's quantiser is folded into that row kernel
// (gnorm_apply_quant_kernel): each warp forms its token's o' row in shared
// memory and quantises it with the standalone quantiser's row routine, so the
// codes are the same and o' never goes to HBM.
//
// Work split. A CTA owns CC channels of one sequence and walks that
// sequence's chunks of TC = 128 steps in order, carrying the state from one
// chunk to the next, so no CTA ever waits for another. A TMA ring keeps the
// next chunks' three gate tiles (CC channels x TC steps each) in flight while
// the current one is computed. Warp w (of 16) owns steps [8w, 8w + 8) of every
// chunk; a lane owns two adjacent channels, in packed fp32 pairs (the f32x2
// instructions of sm_100a). With CC = 64 the 32 lanes cover the 64 channels
// and each lane takes the warp's 8 steps; with CC = 32, 16 lanes cover the
// channels and the two halves of the warp take 4 steps each, which halves the
// registers a thread keeps, so two CTAs share an SM. Within a chunk:
//   1. each lane computes the gates of its steps, keeps f, b = (1 - f) c and
//      g in registers and composes its steps into one affine map
//      h -> A h + B (maps compose: (f2, b2) o (f1, b1) = (f2 f1, f2 b1 + b2));
//      with CC = 32 the two halves' maps are combined through a shuffle;
//   2. the warps' maps meet in shared memory (one barrier per chunk); each
//      warp folds the maps before it onto the chunk's entering state, and the
//      last warp also gets the state leaving the chunk;
//   3. each lane replays its steps from its entering state and stores o'.
// The maps and the leaving state are double-buffered by chunk parity, so a
// warp may start the next chunk while others still fold this one; the stage
// is free for the next copy once every warp is past the barrier (only step 1
// reads it). Every wait on the ring is bounded: on timeout the kernel records
// status code 2 and returns (its output is then invalid; mmf_check reports
// MMF_ERR_TIMEOUT).
#include <type_traits>

#include "kernels.cuh"
#include "quant_row.cuh"
#include "tma.cuh"

namespace mmf {

namespace {

constexpr int TC = 128;         // steps per chunk
constexpr int SW = 16;          // warps per CTA
constexpr int WS = TC / SW;     // steps per warp
constexpr int kThreads = SW * 32;
constexpr int kMaxStages = 4;

// Two channels at once in packed fp32 pairs: lane values x (low word) and y
// (high word).
struct F2 {
  unsigned long long v;
};

// Shared memory: this header, then the ring of `nst` stages of
// T [3][TC][CC] (gate f, c, g x step x channel) at a 128-byte boundary.
template <int CC>
struct ScanSmem {
  static constexpr int NP = CC / 2;     // channel pairs
  F2 A[2][SW][NP];                      // [chunk parity][warp][pair]: composed multiplier of the warp's steps
  F2 Bv[2][SW][NP];                     //   and composed offset
  F2 hnext[2][NP];                      // [chunk parity]: state leaving the chunk (written by the last warp)
  uint64_t full[kMaxStages];
};
template <int CC> constexpr size_t tiles_offset() { return (sizeof(ScanSmem<CC>) + 127) / 128 * 128; }

// hardware approximations (special-function unit): 2^x and 1/x, subnormals flushed
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kMinZ = -29.0f;   // pre-activations are raised to at least -29 (e^-z <= e^29)

// packing and unpacking are register-pair moves (no arithmetic)
__device__ __forceinline__ F2 f2(float x, float y) {
  F2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(x), "f"(y));
  return r;
}
__device__ __forceinline__ float lo(F2 a) {
  float x;
  asm("{ .reg .f32 t; mov.b64 {%0, t}, %1; }" : "=f"(x) : "l"(a.v));
  return x;
}
__device__ __forceinline__ float hi(F2 a) {
  float y;
  asm("{ .reg .f32 t; mov.b64 {t, %0}, %1; }" : "=f"(y) : "l"(a.v));
  return y;
}
__device__ __forceinline__ F2 fma2(F2 a, F2 b, F2 c) {
  F2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d.v) : "l"(a.v), "l"(b.v), "l"(c.v));
  return d;
}
__device__ __forceinline__ F2 mul2(F2 a, F2 b) {
  F2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d.v) : "l"(a.v), "l"(b.v));
  return d;
}
__device__ __forceinline__ F2 add2(F2 a, F2 b) {
  F2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d.v) : "l"(a.v), "l"(b.v));
  return d;
}
__device__ __forceinline__ F2 shfl2(F2 a, int src) { return F2{__shfl_sync(0xffffffffu, a.v, src)}; }

// A channel pair of one gate, as fp32, raised to at least kMinZ (NaN stays
// NaN). bf16: one packed max on the two raw halves, then the exact widening.
__device__ __forceinline__ F2 load_z(const bf16* p) {
  uint32_t w = *reinterpret_cast<const uint32_t*>(p);
  asm("max.NaN.bf16x2 %0, %0, %1;" : "+r"(w) : "r"(0xC1E8C1E8u));   // bf16 -29.0 in both halves
  return f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ F2 load_z(const float* p) {
  const float2 v = *reinterpret_cast<const float2*>(p);   // NaN stays NaN
  return f2(v.x < kMinZ ? kMinZ : v.x, v.y < kMinZ ? kMinZ : v.y);
}
__device__ __forceinline__ F2 load_h(const float* p) { return F2{*reinterpret_cast<const unsigned long long*>(p)}; }
__device__ __forceinline__ void store_pair(bf16* p, F2 v) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(lo(v), hi(v));
}
__device__ __forceinline__ void store_pair(float* p, F2 v) { *reinterpret_cast<unsigned long long*>(p) = v.v; }

__device__ __forceinline__ F2 exp_neg(F2 z) {   // e^-z per lane (z >= -29, so at most e^29)
  const F2 t = mul2(z, f2(-kLog2e, -kLog2e));
  return f2(ex2_approx(lo(t)), ex2_approx(hi(t)));
}

// The three logistic terms of a channel pair with one reciprocal per channel:
// with E_x = e^-x, p_x = 1 + E_x and r = 1 / (p_f p_c p_g),
//   f = sigmoid(zf) = p_c p_g r,   g = sigmoid(zg) = p_f p_c r,
//   b = (1 - f) SiLU(zc) = zc (E_f / p_f)(1 / p_c) = zc E_f p_g r.
// Every z is at least -29 (see load_z), so the product stays finite
// ((1 + e^29)^3 < 2^127); below -29 a logistic is under 3e-13 and the floor
// moves it by less than that.
// With SWISH the third term is the swish gate g = zg sigmoid(zg) = zg p_f p_c r.
template <bool SWISH>
__device__ __forceinline__ void gates2(F2 zf, F2 zc, F2 zg, F2& f, F2& b, F2& g) {
  const F2 one = f2(1.0f, 1.0f);
  const F2 ef = exp_neg(zf);
  const F2 pf = add2(ef, one);
  const F2 pc = add2(exp_neg(zc), one);
  const F2 pg = add2(exp_neg(zg), one);
  const F2 pfc = mul2(pf, pc);
  const F2 pp = mul2(pfc, pg);
  const F2 r = f2(rcp_approx(lo(pp)), rcp_approx(hi(pp)));
  f = mul2(mul2(pc, pg), r);
  g = SWISH ? mul2(zg, mul2(pfc, r)) : mul2(pfc, r);
  b = mul2(mul2(mul2(zc, ef), pg), r);
}

// Sums of q[k] (one value per step k of the lane) over the NP lanes of the
// lane's step group. Reduce-scatter by halving: at offset NP/2 a lane keeps the
// half of its steps picked by that lane bit and adds its partner's copy of it,
// and so on down to one value at offset NP/LS; plain xor-adds over the lower
// offsets finish the sum. Returns the total of step (lane % NP) / (NP / LS),
// log2(LS) + log2(NP / LS) rounds and LS - 1 + log2(NP / LS) shuffles.
template <int NP, int LS>
__device__ __forceinline__ float group_step_sum(float (&q)[LS], int lane) {
#pragma unroll
  for (int n = LS, o = NP / 2; n > 1; n >>= 1, o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float keep = up ? q[i + n / 2] : q[i];
      const float send = up ? q[i] : q[i + n / 2];
      q[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float t = q[0];
#pragma unroll
  for (int o = NP / LS / 2; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}



// Bounded wait for a stage's copies after a timeout, so none lands once the CTA is gone.
__device__ void drain_stage(uint64_t* bar, uint32_t parity, long long limit) {
  const long long t_start = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t_start < limit) {
  }
}

// CC = 32 keeps at most 64 registers per thread so that two CTAs share an SM.
// GN: g_norm mode; `o` receives v = swish(g~) h in fp32 and `ss` [B*T_][n_cb]
// the partial sums of h^2 (see the file comment). Otherwise `o` receives o'.
// HS: `ss` receives the states h_t themselves in fp32 (what the backward pass
// reads), and `o` (o') may be null.
template <typename T, int CC, bool GN, bool HS = false>
__global__ void __launch_bounds__(kThreads, 64 / CC)
    mlgru_scan_kernel(const __grid_constant__ CUtensorMap map, int B, int T_, int d, int n_cb, int nst,
                      float* __restrict__ h, void* __restrict__ out, float* __restrict__ ss, int* status,
                      long long wait_cycles, int skip_chunk) {
  using OT = std::conditional_t<GN, float, T>;
  OT* __restrict__ o = static_cast<OT*>(out);
  using S = ScanSmem<CC>;
  constexpr int NP = S::NP;         // channel pairs: lanes per step group
  constexpr int H = 32 / NP;        // lane groups splitting the warp's steps (1 or 2)
  constexpr int LS = WS / H;        // steps per lane
  using Tile = T[3][TC][CC];
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  S& sm = *reinterpret_cast<S*>(base);
  Tile* ring = reinterpret_cast<Tile*>(base + tiles_offset<CC>());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pr = lane % NP, grp = lane / NP;   // channel pair, step group
  const int b = blockIdx.x / n_cb, cb = blockIdx.x - b * n_cb;
  const int ch = cb * CC + 2 * pr;
  const bool valid = ch < d;           // d % 8 == 0: the pair is all in or all out
  const int nchunk = ceil_div(T_, TC);
  const int tw = warp * WS + grp * LS;   // the lane's first step within a chunk
  constexpr uint32_t kChunkBytes = 3u * TC * CC * sizeof(T);

  auto issue = [&](int j) {   // thread 0: the three gate tiles of chunk j into stage j % nst
    const int s = j % nst;
    if (j == skip_chunk && blockIdx.x == 0) return;   // test hook: this copy is never issued
    mbar_arrive_expect_tx(&sm.full[s], kChunkBytes);
    for (int g = 0; g < 3; ++g) tma_load_2d(&ring[s][g][0][0], &map, g * d + cb * CC, b * T_ + j * TC, &sm.full[s]);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&sm.full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&map);
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();   // the pre-activations and the state are the previous kernels' output
  if (threadIdx.x == 0)
    for (int j = 0; j < nst && j < nchunk; ++j) issue(j);
  F2 hin = f2(0.0f, 0.0f);   // state entering the chunk (chunk 0: the carried state)
  if (valid) hin = load_h(h + (size_t)b * d + ch);

  for (int j = 0; j < nchunk; ++j) {
    const int s = j % nst, par = j & 1;
    bool got = mbar_try_wait(&sm.full[s], (uint32_t)(j / nst) & 1u);
    if (!got) {
      const long long t_start = clock64();
      while (!(got = mbar_try_wait(&sm.full[s], (uint32_t)(j / nst) & 1u)) && clock64() - t_start < wait_cycles) {
      }
    }
    const int t0 = j * TC;
    const T(*tile)[TC][CC] = ring[s];
    const bool full = t0 + TC <= T_;   // every step of the chunk is inside the sequence
    // 1. gates and this lane's composed map (a timed-out stage gives garbage, never used)
    F2 f[LS], bb[LS], gg[LS];
    F2 Aa = f2(1.0f, 1.0f), Bb = f2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < LS; ++k) {
      const int tl = tw + k;
      if (full || t0 + tl < T_) {
        gates2<GN>(load_z(&tile[0][tl][2 * pr]), load_z(&tile[1][tl][2 * pr]), load_z(&tile[2][tl][2 * pr]), f[k],
                   bb[k], gg[k]);
      } else {   // past the end of the sequence: identity map
        f[k] = f2(1.0f, 1.0f);
        bb[k] = f2(0.0f, 0.0f);
        gg[k] = f2(0.0f, 0.0f);
      }
      Bb = fma2(f[k], Bb, bb[k]);
      Aa = mul2(Aa, f[k]);
    }
    F2 A0 = Aa, B0 = Bb;   // the first step group's map (CC = 32)
    if constexpr (H == 2) {
      A0 = shfl2(Aa, pr);
      B0 = shfl2(Bb, pr);
      if (grp == 1) {   // the warp's map: the second group's after the first's
        Bb = fma2(Aa, B0, Bb);
        Aa = mul2(Aa, A0);
      }
    }
    if (grp == H - 1) {
      sm.A[par][warp][pr] = Aa;
      sm.Bv[par][warp][pr] = Bb;
    }
    if (__syncthreads_or(!got)) {   // give up: let the copies in flight land (bounded), then leave
      if (threadIdx.x == 0) {
        if (status) atomicExch(status, 2);
        for (int q = j; q < j + nst && q < nchunk; ++q)
          drain_stage(&sm.full[q % nst], (uint32_t)(q / nst) & 1u, wait_cycles);
      }
      return;
    }
    // every warp is done with the stage: refill it
    if (threadIdx.x == 0 && j + nst < nchunk) {
      fence_proxy_async_smem();
      issue(j + nst);
    }
    // 2. this warp's entering state (the maps of the warps before it); the last
    //    warp also gets the state leaving the chunk
    if (j > 0) hin = sm.hnext[par ^ 1][pr];
    F2 hw = hin;
    for (int w = 0; w < warp; ++w) hw = fma2(sm.A[par][w][pr], hw, sm.Bv[par][w][pr]);
    if (warp == SW - 1 && grp == H - 1) sm.hnext[par][pr] = fma2(Aa, hw, Bb);
    if constexpr (H == 2) {
      if (grp == 1) hw = fma2(A0, hw, B0);
    }
    // 3. replay this lane's steps and store o' (GN: v and the squares' partial sums)
    float sq[LS];
    if (valid) {
      const size_t e0 = ((size_t)b * T_ + t0 + tw) * d + ch;
#pragma unroll
      for (int k = 0; k < LS; ++k) {
        hw = fma2(f[k], hw, bb[k]);
        if (full || t0 + tw + k < T_) {
          if (!HS || o != nullptr) store_pair(o + e0 + (size_t)k * d, mul2(gg[k], hw));
          if constexpr (HS) store_pair(ss + e0 + (size_t)k * d, hw);
        }
        if constexpr (GN) {
          const F2 h2 = mul2(hw, hw);
          sq[k] = lo(h2) + hi(h2);
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < LS; ++k) sq[k] = 0.0f;
    }
    if constexpr (GN) {
      const float tot = group_step_sum<NP, LS>(sq, lane);
      const int k = (lane % NP) / (NP / LS);   // the step whose total this lane holds
      if (lane % (NP / LS) == 0 && (full || t0 + tw + k < T_))
        ss[((size_t)b * T_ + t0 + tw + k) * n_cb + cb] = tot;
    }
  }
  __syncthreads();   // the last warp has written the state leaving the last chunk
  if (valid && warp == 0 && grp == 0) {
    const F2 hl = sm.hnext[(nchunk - 1) & 1][pr];
    store_pair(h + (size_t)b * d + ch, hl);
  }
}

template <typename T, int CC, bool GN, bool HS = false>
cudaError_t launch_typed(const void* pre, int B, int T_, int d, float* h, void* o, float* ss, int* status,
                         long long wait_cycles, int skip_chunk, cudaStream_t stream) {
  CUtensorMap map;
  const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  // box = one gate of one chunk (CC channels x TC steps); a stage holds 3 boxes
  if (!make_tma_2d(&map, pre, dt, (int)sizeof(T), (uint64_t)3 * d, (uint64_t)B * T_, CC, TC,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const int n_cb = ceil_div(d, CC);
  const size_t stage_bytes = sizeof(T) * 3 * TC * CC;
  const size_t budget = CC == 32 ? 96 * 1024 : 192 * 1024;   // two CTAs per SM with CC = 32
  const int nst = (int)std::max<size_t>(2, std::min<size_t>(kMaxStages, budget / stage_bytes));
  const size_t smem = 128 + tiles_offset<CC>() + nst * stage_bytes;
  auto kern = mlgru_scan_kernel<T, CC, GN, HS>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(B * n_cb), dim3(kThreads), smem, stream, map, B, T_, d, n_cb, nst, h, o, ss, status,
                    wait_cycles, skip_chunk);
}

// o'[m, :] = v[m, :] * (1 / sqrt(sum_c ss[m, c] / d + eps)) * gain, one warp per
// token row, four channels per lane per step (16-byte loads of v and gain).
template <typename T>
__global__ void __launch_bounds__(256) gnorm_apply_kernel(const float* __restrict__ v, const float* __restrict__ ss,
                                                          int n_cb, const float* __restrict__ gain, float eps, int M,
                                                          int d, T* __restrict__ o) {
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (blockDim.x >> 5);
  pdl_trigger();
  pdl_wait();   // v and ss are the scan's output
  for (int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); m < M; m += nw) {
    float t = 0.0f;
    for (int c = lane; c < n_cb; c += 32) t += ss[(size_t)m * n_cb + c];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    const float rinv = __frsqrt_rn(__fadd_rn(__fdiv_rn(t, (float)d), eps));
    const float4* vr = reinterpret_cast<const float4*>(v + (size_t)m * d);
    const float4* gr = reinterpret_cast<const float4*>(gain);
    T* orow = o + (size_t)m * d;
    for (int k = lane; k < d / 4; k += 32) {
      const float4 x = vr[k], g = gr[k];
      const float y0 = x.x * rinv * g.x, y1 = x.y * rinv * g.y, y2 = x.z * rinv * g.z, y3 = x.w * rinv * g.w;
      if constexpr (sizeof(T) == 2) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(y0, y1), b = __floats2bfloat162_rn(y2, y3);
        uint2 w;
        w.x = *reinterpret_cast<const uint32_t*>(&a);
        w.y = *reinterpret_cast<const uint32_t*>(&b);
        *reinterpret_cast<uint2*>(orow + 4 * k) = w;
      } else {
        *reinterpret_cast<float4*>(orow + 4 * k) = make_float4(y0, y1, y2, y3);
      }
    }
  }
}

// gnorm_apply_kernel's o' row, then the o projection's RMSNorm + absmax
// quantisation of it (quant_row, the standalone quantiser's routine and fp32
// steps) from a per-warp shared-memory copy of the row; o' itself goes to HBM
// only when `o` is given. One warp per token row.
constexpr int kApplyWarps = 8;
template <typename T, bool GAIN>
__global__ void __launch_bounds__(kApplyWarps * 32)
    gnorm_apply_quant_kernel(const float* __restrict__ v, const float* __restrict__ ss, int n_cb,
                             const float* __restrict__ gain, float eps_g, int M, int d, T* __restrict__ o,
                             const float* __restrict__ qgain, float eps, int8_t* __restrict__ q,
                             float* __restrict__ scale, int32_t* __restrict__ qsum, int pitch) {
  extern __shared__ uint4 rows[];   // [kApplyWarps][pitch / 16]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  T* row_sm = reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(rows) + (size_t)warp * pitch);
  const int nw = gridDim.x * kApplyWarps;
  const int nvec = d * (int)sizeof(T) / 16;
  pdl_trigger();
  pdl_wait();   // v and ss are the scan's output
  for (int m = blockIdx.x * kApplyWarps + warp; m < M; m += nw) {
    float t = 0.0f;
    for (int c = lane; c < n_cb; c += 32) t += ss[(size_t)m * n_cb + c];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    const float rinv = __frsqrt_rn(__fadd_rn(__fdiv_rn(t, (float)d), eps_g));
    const float4* vr = reinterpret_cast<const float4*>(v + (size_t)m * d);
    const float4* gr = reinterpret_cast<const float4*>(gain);
#pragma unroll 4
    for (int k = lane; k < d / 4; k += 32) {
      const float4 x = vr[k], g = gr[k];
      const float y0 = x.x * rinv * g.x, y1 = x.y * rinv * g.y, y2 = x.z * rinv * g.z, y3 = x.w * rinv * g.w;
      if constexpr (sizeof(T) == 2) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(y0, y1), b = __floats2bfloat162_rn(y2, y3);
        uint2 w;
        w.x = *reinterpret_cast<const uint32_t*>(&a);
        w.y = *reinterpret_cast<const uint32_t*>(&b);
        *reinterpret_cast<uint2*>(row_sm + 4 * k) = w;
        if (o) *reinterpret_cast<uint2*>(o + (size_t)m * d + 4 * k) = w;
      } else {
        const float4 w = make_float4(y0, y1, y2, y3);
        *reinterpret_cast<float4*>(row_sm + 4 * k) = w;
        if (o) *reinterpret_cast<float4*>(o + (size_t)m * d + 4 * k) = w;
      }
    }
    __syncwarp();
    const RowCode rc = quant_row<T, GAIN, false>(reinterpret_cast<const uint4*>(row_sm), nvec, d, qgain, eps,
                                                 q + (size_t)m * d, lane);
    if (lane == 0) {
      scale[m] = rc.scale;
      qsum[m] = rc.qsum;
    }
    __syncwarp();   // the row buffer is rewritten for the next row
  }
}

// ---------------------------------------------------------------- backward
// The exact derivative of the recurrence above for upstream gradients
// do = dL/do' and dhT = dL/dh_T. With lambda_t = dL/dh_t and mu_t = f_t lambda_t
// (the part of lambda_t that reaches h_{t-1}):
//   lambda_t = do_t g_t + mu_{t+1},   mu_t = f_t lambda_t,   mu_T = dhT
//   dg~_t = do_t h_t g_t (1 - g_t)
//   df~_t = lambda_t (h_{t-1} - c_t) f_t (1 - f_t)
//   dc~_t = lambda_t (1 - f_t) sigmoid(c~_t) (1 + c~_t (1 - sigmoid(c~_t)))
//   dh0 = mu_0
// mu runs backwards through affine maps mu -> f_t mu + f_t do_t g_t, which
// compose like the forward maps. One CTA per (sequence, 64 channels) walks the
// chunks from the last to the first; within a chunk each lane composes its 8
// steps, the warps' maps meet in shared memory (one barrier per chunk, double
// buffered by chunk parity), each warp folds the maps of the warps after it
// onto the mu entering the chunk's end, then replays its steps backwards and
// stores the three gradients. The states h_t come from the forward scan in its
// HS mode (fp32). This form reads its inputs with plain loads and an L2
// prefetch of the next chunk (fp32 runs, whose tiles would not fit twice in
// shared memory); bf16 runs take the TMA-staged form below.
constexpr int kBwdCC = 64;
struct BwdSmem {
  F2 A[2][SW][kBwdCC / 2];
  F2 Bv[2][SW][kBwdCC / 2];
  F2 mu_prev[2][kBwdCC / 2];   // mu leaving the chunk at its start (written by warp 0)
};

__device__ __forceinline__ F2 load_zr(const bf16* p) {   // raw value pair (no floor)
  const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
  return f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ F2 load_zr(const float* p) { return F2{*reinterpret_cast<const unsigned long long*>(p)}; }

// sigmoid of a pair, with the exponent argument floored as in the forward pass
__device__ __forceinline__ F2 sigmoid2(F2 z) {
  const F2 zc = f2(fmaxf(lo(z), kMinZ), fmaxf(hi(z), kMinZ));
  const F2 p = add2(exp_neg(zc), f2(1.0f, 1.0f));
  return f2(rcp_approx(lo(p)), rcp_approx(hi(p)));
}

// L2 prefetch of chunk j's rows of this CTA's channels (pre-activations, dL/do',
// states): one 128-byte line per thread and step of the loop.
template <typename T>
__device__ __forceinline__ void bwd_prefetch(const T* pre, const float* hs, const T* dout, size_t row0, int T_, int d,
                                             int ch0, int j) {
  constexpr int kLineEl = 128 / sizeof(T);        // elements of T per line
  constexpr int kPerRowT = kBwdCC / kLineEl;      // lines per row of T (1 or 2)
  constexpr int kPerRowH = kBwdCC * 4 / 128;      // lines per row of fp32 states (2)
  constexpr int kLines = TC * (4 * kPerRowT + kPerRowH);
  for (int l = threadIdx.x; l < kLines; l += kThreads) {
    int r, idx = l;
    const void* addr;
    if (idx < TC * 3 * kPerRowT) {   // pre-activations: row, gate, part
      r = idx / (3 * kPerRowT);
      const int rem = idx - r * 3 * kPerRowT, g = rem / kPerRowT, part = rem - g * kPerRowT;
      if (j * TC + r >= T_ || ch0 + part * kLineEl >= d) continue;   // the line starts inside the row
      addr = pre + ((row0 + j * TC + r) * 3 + g) * (size_t)d + ch0 + part * kLineEl;
    } else if ((idx -= TC * 3 * kPerRowT) < TC * kPerRowT) {   // dL/do'
      r = idx / kPerRowT;
      if (j * TC + r >= T_ || ch0 + (idx - r * kPerRowT) * kLineEl >= d) continue;
      addr = dout + (row0 + j * TC + r) * (size_t)d + ch0 + (idx - r * kPerRowT) * kLineEl;
    } else {   // states
      idx -= TC * kPerRowT;
      r = idx / kPerRowH;
      if (j * TC + r >= T_ || ch0 + (idx - r * kPerRowH) * 32 >= d) continue;
      addr = hs + (row0 + j * TC + r) * (size_t)d + ch0 + (idx - r * kPerRowH) * 32;
    }
    asm volatile("prefetch.global.L2 [%0];" ::"l"(addr));
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    mlgru_scan_bwd_kernel(const T* __restrict__ pre, const float* __restrict__ hs, const float* __restrict__ h0,
                          const T* __restrict__ dout, const float* __restrict__ dhT, int B, int T_, int d, int n_cb,
                          T* __restrict__ dpre, float* __restrict__ dh0) {
  __shared__ BwdSmem sm;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x / n_cb, cb = blockIdx.x - b * n_cb;
  const int ch = cb * kBwdCC + 2 * lane;
  const bool valid = ch < d;
  const int nchunk = ceil_div(T_, TC);
  const int tw = warp * WS;
  pdl_trigger();
  pdl_wait();   // the states are the forward scan's output
  F2 mu_end = f2(0.0f, 0.0f);   // mu entering the current chunk's end
  if (valid && dhT != nullptr) mu_end = load_h(dhT + (size_t)b * d + ch);
  const size_t row0 = (size_t)b * T_;
  const int ch0 = cb * kBwdCC;
  bwd_prefetch(pre, hs, dout, row0, T_, d, ch0, nchunk - 1);
  for (int j = nchunk - 1; j >= 0; --j) {
    const int par = j & 1;
    const int t0 = j * TC;
    if (j > 0) bwd_prefetch(pre, hs, dout, row0, T_, d, ch0, j - 1);   // the next chunk, into L2
    // 1. f_t and a_t = do_t g_t of this lane's steps, composed backwards
    F2 f[WS], a[WS];
    F2 Aa = f2(1.0f, 1.0f), Bb = f2(0.0f, 0.0f);
#pragma unroll
    for (int k = WS - 1; k >= 0; --k) {
      const int t = t0 + tw + k;
      if (valid && t < T_) {
        const T* pr = pre + (row0 + t) * 3 * (size_t)d + ch;
        f[k] = sigmoid2(load_zr(pr));
        const F2 g = sigmoid2(load_zr(pr + 2 * (size_t)d));
        a[k] = mul2(load_zr(dout + (row0 + t) * (size_t)d + ch), g);
      } else {   // past the end of the sequence (or channel): identity map
        f[k] = f2(1.0f, 1.0f);
        a[k] = f2(0.0f, 0.0f);
      }
      // step k after the steps behind it: mu -> f (a + (A mu + B))
      Bb = mul2(f[k], add2(a[k], Bb));
      Aa = mul2(f[k], Aa);
    }
    sm.A[par][warp][lane] = Aa;
    sm.Bv[par][warp][lane] = Bb;
    __syncthreads();
    // 2. mu entering this warp's last step: the maps of the warps after it,
    //    applied to the mu entering the chunk's end; warp 0 also gets the mu
    //    leaving the chunk's start
    if (j < nchunk - 1) mu_end = sm.mu_prev[par ^ 1][lane];
    F2 mu = mu_end;
    for (int w = SW - 1; w > warp; --w) mu = fma2(sm.A[par][w][lane], mu, sm.Bv[par][w][lane]);
    if (warp == 0) sm.mu_prev[par][lane] = fma2(Aa, mu, Bb);
    // 3. replay backwards: lambda, the three gradients, mu for the step before
#pragma unroll
    for (int k = WS - 1; k >= 0; --k) {
      const int t = t0 + tw + k;
      const F2 lam = add2(a[k], mu);
      if (valid && t < T_) {
        const T* pr = pre + (row0 + t) * 3 * (size_t)d + ch;
        const F2 zc = load_zr(pr + d);
        const F2 g = sigmoid2(load_zr(pr + 2 * (size_t)d));
        const F2 sc = sigmoid2(zc);
        const F2 one = f2(1.0f, 1.0f);
        const F2 c = mul2(zc, sc);
        const F2 ht = load_h(hs + (row0 + t) * (size_t)d + ch);
        const F2 hp = t > 0 ? load_h(hs + (row0 + t - 1) * (size_t)d + ch) : load_h(h0 + (size_t)b * d + ch);
        const F2 dov = load_zr(dout + (row0 + t) * (size_t)d + ch);
        const F2 omf = add2(one, mul2(f[k], f2(-1.0f, -1.0f)));
        const F2 omg = add2(one, mul2(g, f2(-1.0f, -1.0f)));
        const F2 dzg = mul2(mul2(dov, ht), mul2(g, omg));
        const F2 dzf = mul2(mul2(lam, add2(hp, mul2(c, f2(-1.0f, -1.0f)))), mul2(f[k], omf));
        const F2 silu_p = mul2(sc, fma2(zc, add2(one, mul2(sc, f2(-1.0f, -1.0f))), one));
        const F2 dzc = mul2(mul2(lam, omf), silu_p);
        T* out = dpre + (row0 + t) * 3 * (size_t)d + ch;
        store_pair(out, dzf);
        store_pair(out + d, dzc);
        store_pair(out + 2 * (size_t)d, dzg);
      }
      mu = mul2(f[k], lam);
    }
  }
  __syncthreads();   // warp 0 has written the mu leaving the first chunk
  if (valid && warp == 0) store_pair(dh0 + (size_t)b * d + ch, sm.mu_prev[0][lane]);
}

// The same backward for bf16 with its inputs staged by TMA: each chunk's
// pre-activation, dL/do' and state tiles (96 KB) land in one of two stages, so
// phases 1 and 3 read shared memory; a stage is refilled with the chunk two
// ahead at the next chunk's barrier, when every warp has finished its replay.
// Every wait is bounded (status code 2 on timeout, as in the forward scan).
struct BwdTile {
  bf16 pre[3][TC][kBwdCC];
  bf16 dout[TC][kBwdCC];
  float h[TC][kBwdCC];
};
constexpr uint32_t kBwdTileBytes = sizeof(BwdTile);

__global__ void __launch_bounds__(kThreads, 1)
    mlgru_scan_bwd_tma_kernel(const __grid_constant__ CUtensorMap map_pre, const __grid_constant__ CUtensorMap map_do,
                              const __grid_constant__ CUtensorMap map_h, const float* __restrict__ hs,
                              const float* __restrict__ h0, const float* __restrict__ dhT, int B, int T_, int d,
                              int n_cb, bf16* __restrict__ dpre, float* __restrict__ dh0, int* status,
                              long long wait_cycles, int skip_chunk) {
  __shared__ BwdSmem sm;
  __shared__ uint64_t full[2];
  extern __shared__ uint8_t smem_raw[];
  BwdTile* ring = reinterpret_cast<BwdTile*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x / n_cb, cb = blockIdx.x - b * n_cb;
  const int ch = cb * kBwdCC + 2 * lane;
  const bool valid = ch < d;
  const int nchunk = ceil_div(T_, TC);
  const int tw = warp * WS;
  const size_t row0 = (size_t)b * T_;
  auto issue = [&](int j) {   // thread 0: chunk j into stage (nchunk - 1 - j) & 1
    const int s = (nchunk - 1 - j) & 1;
    const int y = (int)row0 + j * TC;
    if (j == skip_chunk && blockIdx.x == 0) return;   // test hook: this copy is never issued
    mbar_arrive_expect_tx(&full[s], kBwdTileBytes);
    for (int g = 0; g < 3; ++g) tma_load_2d(&ring[s].pre[g][0][0], &map_pre, g * d + cb * kBwdCC, y, &full[s]);
    tma_load_2d(&ring[s].dout[0][0], &map_do, cb * kBwdCC, y, &full[s]);
    tma_load_2d(&ring[s].h[0][0], &map_h, cb * kBwdCC, y, &full[s]);
  };
  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();   // the states are the forward scan's output
  if (threadIdx.x == 0) {
    issue(nchunk - 1);
    if (nchunk > 1) issue(nchunk - 2);
  }
  F2 mu_end = f2(0.0f, 0.0f);
  if (valid && dhT != nullptr) mu_end = load_h(dhT + (size_t)b * d + ch);
  for (int j = nchunk - 1; j >= 0; --j) {
    const int q = nchunk - 1 - j, s = q & 1, par = j & 1;
    const int t0 = j * TC;
    bool got = mbar_try_wait(&full[s], (uint32_t)(q >> 1) & 1u);
    if (!got) {
      const long long t_start = clock64();
      while (!(got = mbar_try_wait(&full[s], (uint32_t)(q >> 1) & 1u)) && clock64() - t_start < wait_cycles) {
      }
    }
    const BwdTile& tile = ring[s];
    // 1. f_t and a_t = do_t g_t, composed backwards
    F2 f[WS], a[WS];
    F2 Aa = f2(1.0f, 1.0f), Bb = f2(0.0f, 0.0f);
#pragma unroll
    for (int k = WS - 1; k >= 0; --k) {
      const int tl = tw + k;
      if (valid && t0 + tl < T_) {
        f[k] = sigmoid2(load_zr(&tile.pre[0][tl][2 * lane]));
        a[k] = mul2(load_zr(&tile.dout[tl][2 * lane]), sigmoid2(load_zr(&tile.pre[2][tl][2 * lane])));
      } else {
        f[k] = f2(1.0f, 1.0f);
        a[k] = f2(0.0f, 0.0f);
      }
      Bb = mul2(f[k], add2(a[k], Bb));
      Aa = mul2(f[k], Aa);
    }
    sm.A[par][warp][lane] = Aa;
    sm.Bv[par][warp][lane] = Bb;
    if (__syncthreads_or(!got)) {   // give up: let the copies in flight land (bounded), then leave
      if (threadIdx.x == 0) {
        if (status) atomicExch(status, 2);
        for (int qq = q; qq < q + 2 && qq < nchunk; ++qq) drain_stage(&full[qq & 1], (uint32_t)(qq >> 1) & 1u, wait_cycles);
      }
      return;
    }
    // the stage of the chunk before (q - 1) is free: every warp has replayed it
    if (threadIdx.x == 0 && q >= 1 && j - 1 >= 0) {
      fence_proxy_async_smem();
      issue(j - 1);
    }
    // 2. mu entering this warp's last step; warp 0 also the mu leaving the chunk
    if (j < nchunk - 1) mu_end = sm.mu_prev[par ^ 1][lane];
    F2 mu = mu_end;
    for (int w = SW - 1; w > warp; --w) mu = fma2(sm.A[par][w][lane], mu, sm.Bv[par][w][lane]);
    if (warp == 0) sm.mu_prev[par][lane] = fma2(Aa, mu, Bb);
    // 3. replay backwards
#pragma unroll
    for (int k = WS - 1; k >= 0; --k) {
      const int tl = tw + k, t = t0 + tl;
      const F2 lam = add2(a[k], mu);
      if (valid && t < T_) {
        const F2 zc = load_zr(&tile.pre[1][tl][2 * lane]);
        const F2 g = sigmoid2(load_zr(&tile.pre[2][tl][2 * lane]));
        const F2 sc = sigmoid2(zc);
        const F2 one = f2(1.0f, 1.0f), neg = f2(-1.0f, -1.0f);
        const F2 c = mul2(zc, sc);
        const F2 ht = load_h(&tile.h[tl][2 * lane]);
        const F2 hp = tl > 0 ? load_h(&tile.h[tl - 1][2 * lane])
                             : (t > 0 ? load_h(hs + (row0 + t - 1) * (size_t)d + ch) : load_h(h0 + (size_t)b * d + ch));
        const F2 dov = load_zr(&tile.dout[tl][2 * lane]);
        const F2 omf = add2(one, mul2(f[k], neg));
        const F2 omg = add2(one, mul2(g, neg));
        const F2 dzg = mul2(mul2(dov, ht), mul2(g, omg));
        const F2 dzf = mul2(mul2(lam, add2(hp, mul2(c, neg))), mul2(f[k], omf));
        const F2 silu_p = mul2(sc, fma2(zc, add2(one, mul2(sc, neg)), one));
        const F2 dzc = mul2(mul2(lam, omf), silu_p);
        bf16* out = dpre + (row0 + t) * 3 * (size_t)d + ch;
        store_pair(out, dzf);
        store_pair(out + d, dzc);
        store_pair(out + 2 * (size_t)d, dzg);
      }
      mu = mul2(f[k], lam);
    }
  }
  __syncthreads();
  if (valid && warp == 0) store_pair(dh0 + (size_t)b * d + ch, sm.mu_prev[0][lane]);
}

// 64 channels per CTA when that gives enough CTAs to cover the GPU, else 32
bool scan_wide(int B, int d) { return (size_t)B * ceil_div(d, 64) >= (size_t)num_sms() * 3 / 4; }

// The scan in g_norm mode: v and the partial sums into ws; n_cb = channel blocks.
cudaError_t launch_scan_gnorm_part(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, void* ws,
                                   int* status, cudaStream_t stream, float*& v, float*& ss, int& n_cb) {
  const size_t M = (size_t)B * T;
  v = static_cast<float*>(ws);
  ss = reinterpret_cast<float*>(static_cast<char*>(ws) + (M * d * sizeof(float) + 255) / 256 * 256);
  const long long wait = wait_limit_cycles();
  const int skip = test_hook("MMF_SCAN_SKIP_CHUNK");
  const bool wide = scan_wide(B, d);
  n_cb = ceil_div(d, wide ? 64 : 32);
  if (dt == MMF_BF16)
    return wide ? launch_typed<bf16, 64, true>(pre, B, T, d, h, v, ss, status, wait, skip, stream)
                : launch_typed<bf16, 32, true>(pre, B, T, d, h, v, ss, status, wait, skip, stream);
  return wide ? launch_typed<float, 64, true>(pre, B, T, d, h, v, ss, status, wait, skip, stream)
              : launch_typed<float, 32, true>(pre, B, T, d, h, v, ss, status, wait, skip, stream);
}

template <typename T, bool GAIN>
cudaError_t launch_apply_quant(const float* v, const float* ss, int n_cb, const float* gain, float eps_g, int M,
                               int d, void* o, const float* qgain, float eps, int8_t* q, float* scale, int32_t* qsum,
                               cudaStream_t stream) {
  const int pitch = (d * (int)sizeof(T) + 127) / 128 * 128;
  const size_t smem = (size_t)kApplyWarps * pitch;
  auto kern = gnorm_apply_quant_kernel<T, GAIN>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = std::max(1, std::min(ceil_div(M, kApplyWarps), num_sms() * 8));
  return launch_pdl(kern, dim3(grid), dim3(kApplyWarps * 32), smem, stream, v, ss, n_cb, gain, eps_g, M, d,
                    static_cast<T*>(o), qgain, eps, q, scale, qsum, pitch);
}

}  // namespace

size_t mlgru_scan_ws_bytes(int, int, int) { return 256; }

cudaError_t launch_mlgru_scan(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, void* o, int* status,
                              cudaStream_t stream) {
  if (B == 0 || T == 0) return cudaSuccess;
  if (!tma_available()) return cudaErrorNotSupported;
  const long long wait = wait_limit_cycles();
  const int skip = test_hook("MMF_SCAN_SKIP_CHUNK");
  const bool wide = scan_wide(B, d);
  if (dt == MMF_BF16)
    return wide ? launch_typed<bf16, 64, false>(pre, B, T, d, h, o, nullptr, status, wait, skip, stream)
                : launch_typed<bf16, 32, false>(pre, B, T, d, h, o, nullptr, status, wait, skip, stream);
  return wide ? launch_typed<float, 64, false>(pre, B, T, d, h, o, nullptr, status, wait, skip, stream)
              : launch_typed<float, 32, false>(pre, B, T, d, h, o, nullptr, status, wait, skip, stream);
}

size_t mlgru_scan_gnorm_ws_bytes(int B, int T, int d) {
  const size_t M = (size_t)B * T;
  return (M * d * sizeof(float) + 255) / 256 * 256 + M * ceil_div(d, 32) * sizeof(float) + 256;
}

cudaError_t launch_mlgru_scan_gnorm(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, const float* gain,
                                    float eps, void* o, void* ws, int* status, cudaStream_t stream) {
  if (B == 0 || T == 0) return cudaSuccess;
  if (!tma_available()) return cudaErrorNotSupported;
  const size_t M = (size_t)B * T;
  float *v, *ss;
  int n_cb;
  cudaError_t e = launch_scan_gnorm_part(pre, dt, B, T, d, h, ws, status, stream, v, ss, n_cb);
  if (e != cudaSuccess) return e;
  constexpr int kWarpsA = 8;
  const int grid = (int)std::max<size_t>(1, std::min<size_t>((M + kWarpsA - 1) / kWarpsA, (size_t)num_sms() * 8));
  if (dt == MMF_BF16)
    return launch_pdl(gnorm_apply_kernel<bf16>, dim3(grid), dim3(32 * kWarpsA), 0, stream, (const float*)v,
                      (const float*)ss, n_cb, gain, eps, (int)M, d, static_cast<bf16*>(o));
  return launch_pdl(gnorm_apply_kernel<float>, dim3(grid), dim3(32 * kWarpsA), 0, stream, (const float*)v,
                    (const float*)ss, n_cb, gain, eps, (int)M, d, static_cast<float*>(o));
}

size_t mlgru_scan_bwd_ws_bytes(int B, int T, int d) { return ((size_t)B * T * d * sizeof(float) + 255) / 256 * 256; }

cudaError_t launch_mlgru_scan_states(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, void* o, float* hs,
                                     int* status, cudaStream_t stream) {
  if (B == 0 || T == 0) return cudaSuccess;
  if (!tma_available()) return cudaErrorNotSupported;
  const long long wait = wait_limit_cycles();
  const bool wide = scan_wide(B, d);
  if (dt == MMF_BF16)
    return wide ? launch_typed<bf16, 64, false, true>(pre, B, T, d, h, o, hs, status, wait, -1, stream)
                : launch_typed<bf16, 32, false, true>(pre, B, T, d, h, o, hs, status, wait, -1, stream);
  return wide ? launch_typed<float, 64, false, true>(pre, B, T, d, h, o, hs, status, wait, -1, stream)
              : launch_typed<float, 32, false, true>(pre, B, T, d, h, o, hs, status, wait, -1, stream);
}

cudaError_t launch_mlgru_scan_bwd(const void* pre, mmf_dtype dt, int B, int T, int d, const float* h0,
                                  const void* dout, const float* dhT, const float* hs_in, void* dpre, float* dh0,
                                  void* ws, int* status, cudaStream_t stream) {
  if (B == 0 || T == 0) return cudaSuccess;
  if (!tma_available()) return cudaErrorNotSupported;
  cudaError_t e = cudaSuccess;
  const long long wait = wait_limit_cycles();
  const float* hsv = hs_in;
  if (hsv == nullptr) {   // 1. the forward states h_t (fp32) into ws, the carried state starting from h0
    float* hcur = dh0;    // scratch for the forward scan's carried state: dh0 is written last
    e = cudaMemcpyAsync(hcur, h0, sizeof(float) * (size_t)B * d, cudaMemcpyDeviceToDevice, stream);
    if (e != cudaSuccess) return e;
    e = launch_mlgru_scan_states(pre, dt, B, T, d, hcur, nullptr, static_cast<float*>(ws), status, stream);
    if (e != cudaSuccess) return e;
    hsv = static_cast<const float*>(ws);
  }
  // 2. the reverse scan (bf16: inputs staged by TMA)
  const int n_cb = ceil_div(d, kBwdCC);
  if (dt == MMF_BF16) {
    CUtensorMap mp, md, mh;
    if (!make_tma_2d(&mp, pre, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)3 * d, (uint64_t)B * T, kBwdCC, TC,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_tma_2d(&md, dout, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)d, (uint64_t)B * T, kBwdCC, TC,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_tma_2d(&mh, hsv, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)d, (uint64_t)B * T, kBwdCC, TC,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    const size_t smem = 2 * sizeof(BwdTile) + 128;
    e = cudaFuncSetAttribute(mlgru_scan_bwd_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(mlgru_scan_bwd_tma_kernel, dim3(B * n_cb), dim3(kThreads), smem, stream, mp, md, mh,
                      hsv, h0, dhT, B, T, d, n_cb, static_cast<bf16*>(dpre), dh0, status, wait,
                      test_hook("MMF_SCAN_SKIP_CHUNK"));
  }
  return launch_pdl(mlgru_scan_bwd_kernel<float>, dim3(B * n_cb), dim3(kThreads), 0, stream,
                    static_cast<const float*>(pre), hsv, h0, static_cast<const float*>(dout), dhT, B, T, d,
                    n_cb, static_cast<float*>(dpre), dh0);
}

cudaError_t launch_mlgru_scan_gnorm_quant(const void* pre, mmf_dtype dt, int B, int T, int d, float* h,
                                          const float* gain, float eps_g, void* o, void* ws, int* status,
                                          const float* qgain, float eps, int8_t* q, float* scale, int32_t* qsum,
                                          cudaStream_t stream) {
  if (B == 0 || T == 0) return cudaSuccess;
  if (!tma_available()) return cudaErrorNotSupported;
  float *v, *ss;
  int n_cb;
  cudaError_t e = launch_scan_gnorm_part(pre, dt, B, T, d, h, ws, status, stream, v, ss, n_cb);
  if (e != cudaSuccess) return e;
  const int M = B * T;
  if (dt == MMF_BF16)
    return qgain ? launch_apply_quant<bf16, true>(v, ss, n_cb, gain, eps_g, M, d, o, qgain, eps, q, scale, qsum, stream)
                 : launch_apply_quant<bf16, false>(v, ss, n_cb, gain, eps_g, M, d, o, qgain, eps, q, scale, qsum,
                                                   stream);
  return qgain ? launch_apply_quant<float, true>(v, ss, n_cb, gain, eps_g, M, d, o, qgain, eps, q, scale, qsum, stream)
               : launch_apply_quant<float, false>(v, ss, n_cb, gain, eps_g, M, d, o, qgain, eps, q, scale, qsum,
                                                  stream);
}

}  // namespace mmf
