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
// Work split. A CTA owns CC channels of one sequence (CC = 64, or 32 when
// there are too few sequence x channel blocks to fill the GPU) and walks that
// sequence's chunks of TC = 128 steps in order, carrying the state in
// registers from one chunk to the next, so no CTA ever waits for another. A
// TMA ring keeps the next chunks' three gate tiles (CC channels x TC steps
// each) in flight while the current one is computed. Within a chunk:
//   1. warp w (of 16) computes the gates of steps [8w, 8w + 8), keeps f,
//      b = (1 - f) c and g in registers and composes its 8 steps into one
//      affine map h -> A h + B (maps compose: (f2, b2) o (f1, b1) =
//      (f2 f1, f2 b1 + b2));
//   2. the warps' maps meet in shared memory; each warp folds the maps before
//      it onto the chunk's entering state, and every warp also folds all
//      sixteen to get the state leaving the chunk;
//   3. each warp replays its 8 steps from its entering state and stores o'.
// Every wait on the ring is bounded: on timeout the kernel records status code
// 2 and returns (its output is then invalid; mmf_check reports MMF_ERR_TIMEOUT).
#include "kernels.cuh"
#include "tma.cuh"

namespace mmf {

namespace {

constexpr int TC = 128;         // steps per chunk
constexpr int SW = 16;          // warps per CTA
constexpr int LS = TC / SW;     // steps per warp
constexpr int kThreads = SW * 32;
constexpr int kMaxStages = 4;

// Shared memory: this header, then the ring of `nst` stages of
// T [3][TC][CC] (gate f, c, g x step x channel) at a 128-byte boundary.
template <int CC>
struct ScanSmem {
  static constexpr int CPL = CC / 32;   // channels per lane
  float A[SW][CPL][32];                 // composed multiplier of each warp's steps
  float Bv[SW][CPL][32];                // composed offset
  float hnext[CPL][32];                 // state leaving the chunk (written by the last warp)
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
constexpr float kMaxExp2 = 29.0f * kLog2e;   // e^-z capped at e^29

// The three logistic terms of one channel-step with one reciprocal: with
// E_x = e^-x, p_x = 1 + E_x and r = 1 / (p_f p_c p_g),
//   f = sigmoid(zf) = p_c p_g r,   g = sigmoid(zg) = p_f p_c r,
//   b = (1 - f) SiLU(zc) = zc (E_f / p_f)(1 / p_c) = zc E_f p_g r.
// Each exponent is capped at 29 so that the product stays finite
// ((1 + e^29)^3 < 2^127); below -29 a logistic is under 3e-13 and the cap
// moves it by less than that.
__device__ __forceinline__ void gates(float zf, float zc, float zg, float& f, float& b, float& g) {
  const float ef = ex2_approx(fminf(-zf * kLog2e, kMaxExp2));
  const float pf = 1.0f + ef;
  const float pc = 1.0f + ex2_approx(fminf(-zc * kLog2e, kMaxExp2));
  const float pg = 1.0f + ex2_approx(fminf(-zg * kLog2e, kMaxExp2));
  const float pfc = pf * pc;
  const float r = rcp_approx(pfc * pg);
  f = (pc * pg) * r;
  g = pfc * r;
  b = ((zc * ef) * pg) * r;
}

// Two channels at once in packed fp32 pairs (the f32x2 instructions of
// sm_100a): lane values x (low word) and y (high word).
struct F2 {
  unsigned long long v;
};
__device__ __forceinline__ F2 f2(float x, float y) {
  return F2{(unsigned long long)__float_as_uint(x) | ((unsigned long long)__float_as_uint(y) << 32)};
}
__device__ __forceinline__ float lo(F2 a) { return __uint_as_float((uint32_t)a.v); }
__device__ __forceinline__ float hi(F2 a) { return __uint_as_float((uint32_t)(a.v >> 32)); }
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
__device__ __forceinline__ F2 ex2_capped(F2 z) {   // e^-z per lane, exponent capped as in gates()
  const F2 t = mul2(z, f2(-kLog2e, -kLog2e));
  return f2(ex2_approx(fminf(lo(t), kMaxExp2)), ex2_approx(fminf(hi(t), kMaxExp2)));
}
// gates() for a channel pair
__device__ __forceinline__ void gates2(F2 zf, F2 zc, F2 zg, F2& f, F2& b, F2& g) {
  const F2 one = f2(1.0f, 1.0f);
  const F2 ef = ex2_capped(zf);
  const F2 pf = add2(ef, one);
  const F2 pc = add2(ex2_capped(zc), one);
  const F2 pg = add2(ex2_capped(zg), one);
  const F2 pfc = mul2(pf, pc);
  const F2 pp = mul2(pfc, pg);
  const F2 r = f2(rcp_approx(lo(pp)), rcp_approx(hi(pp)));
  f = mul2(mul2(pc, pg), r);
  g = mul2(pfc, r);
  b = mul2(mul2(mul2(zc, ef), pg), r);
}
__device__ __forceinline__ F2 load_pair(const bf16* p) {   // two bf16 -> fp32 pair (exact)
  const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
  return F2{(unsigned long long)(w << 16) | ((unsigned long long)(w & 0xffff0000u) << 32)};
}
__device__ __forceinline__ F2 load_pair(const float* p) { return F2{*reinterpret_cast<const unsigned long long*>(p)}; }
__device__ __forceinline__ void store_pair(bf16* p, F2 v) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(lo(v), hi(v));
}
__device__ __forceinline__ void store_pair(float* p, F2 v) { *reinterpret_cast<unsigned long long*>(p) = v.v; }

template <int CPL> struct Lane;
template <> struct Lane<2> {   // two adjacent channels per lane
  __device__ __forceinline__ static void load(const bf16* p, float (&v)[2]) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    v[0] = f.x;
    v[1] = f.y;
  }
  __device__ __forceinline__ static void load(const float* p, float (&v)[2]) {
    const float2 f = *reinterpret_cast<const float2*>(p);
    v[0] = f.x;
    v[1] = f.y;
  }
  __device__ __forceinline__ static void store(bf16* p, const float (&v)[2]) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v[0], v[1]);
  }
  __device__ __forceinline__ static void store(float* p, const float (&v)[2]) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  }
};
template <> struct Lane<1> {   // one channel per lane
  template <typename T> __device__ __forceinline__ static void load(const T* p, float (&v)[1]) { v[0] = to_f32(*p); }
  template <typename T> __device__ __forceinline__ static void store(T* p, const float (&v)[1]) {
    *p = from_f32<T>(v[0]);
  }
};

// Bounded wait for a stage's copies after a timeout, so none lands once the CTA is gone.
__device__ void drain_stage(uint64_t* bar, uint32_t parity, long long limit) {
  const long long t_start = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t_start < limit) {
  }
}

template <typename T, int CC>
__global__ void __launch_bounds__(kThreads, 1)
    mlgru_scan_kernel(const __grid_constant__ CUtensorMap map, int B, int T_, int d, int n_cb, int nst,
                      float* __restrict__ h, T* __restrict__ o, int* status, long long wait_cycles, int skip_chunk) {
  using S = ScanSmem<CC>;
  constexpr int CPL = S::CPL;
  using LN = Lane<CPL>;
  using Tile = T[3][TC][CC];
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  S& sm = *reinterpret_cast<S*>(base);
  Tile* ring = reinterpret_cast<Tile*>(base + tiles_offset<CC>());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x / n_cb, cb = blockIdx.x - b * n_cb;
  const int ch = cb * CC + lane * CPL;
  const bool valid = ch < d;           // d % 8 == 0 and CPL <= 2: the lane's channels are all in or all out
  const int nchunk = ceil_div(T_, TC);
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
  float hin[CPL];
  {
    float z[CPL] = {};
    if (valid) LN::load(h + (size_t)b * d + ch, z);
#pragma unroll
    for (int c = 0; c < CPL; ++c) hin[c] = z[c];
  }

  for (int j = 0; j < nchunk; ++j) {
    const int s = j % nst;
    bool got = mbar_try_wait(&sm.full[s], (uint32_t)(j / nst) & 1u);
    if (!got) {
      const long long t_start = clock64();
      while (!(got = mbar_try_wait(&sm.full[s], (uint32_t)(j / nst) & 1u)) && clock64() - t_start < wait_cycles) {
      }
    }
    if (__syncthreads_or(!got)) {   // give up: let the copies in flight land (bounded), then leave
      if (threadIdx.x == 0) {
        if (status) atomicExch(status, 2);
        for (int q = j; q < j + nst && q < nchunk; ++q)
          drain_stage(&sm.full[q % nst], (uint32_t)(q / nst) & 1u, wait_cycles);
      }
      return;
    }
    const int t0 = j * TC;
    const T(*tile)[TC][CC] = ring[s];
    const bool full = t0 + TC <= T_;   // every step of the chunk is inside the sequence
    T* op = o + ((size_t)b * T_ + t0 + warp * LS) * d + ch;
    if constexpr (CPL == 2) {
      // 1. gates and this warp's composed map, two channels per lane in packed pairs
      F2 f[LS], bb[LS], gg[LS];
      F2 Aa = f2(1.0f, 1.0f), Bb = f2(0.0f, 0.0f);
#pragma unroll
      for (int k = 0; k < LS; ++k) {
        const int tl = warp * LS + k;
        if (full || t0 + tl < T_) {
          gates2(load_pair(&tile[0][tl][2 * lane]), load_pair(&tile[1][tl][2 * lane]),
                 load_pair(&tile[2][tl][2 * lane]), f[k], bb[k], gg[k]);
        } else {   // past the end of the sequence: identity map
          f[k] = f2(1.0f, 1.0f);
          bb[k] = f2(0.0f, 0.0f);
          gg[k] = f2(0.0f, 0.0f);
        }
        Bb = fma2(f[k], Bb, bb[k]);
        Aa = mul2(Aa, f[k]);
      }
      sm.A[warp][0][lane] = lo(Aa);
      sm.A[warp][1][lane] = hi(Aa);
      sm.Bv[warp][0][lane] = lo(Bb);
      sm.Bv[warp][1][lane] = hi(Bb);
      __syncthreads();
      // 2. this warp's entering state (the maps of the warps before it); the
      //    last warp also gets the state leaving the chunk
      F2 hw = f2(hin[0], hin[1]);
      for (int w = 0; w < warp; ++w)
        hw = fma2(f2(sm.A[w][0][lane], sm.A[w][1][lane]), hw, f2(sm.Bv[w][0][lane], sm.Bv[w][1][lane]));
      if (warp == SW - 1) {
        const F2 hn = fma2(Aa, hw, Bb);
        sm.hnext[0][lane] = lo(hn);
        sm.hnext[1][lane] = hi(hn);
      }
      // 3. replay this warp's steps and store o'
      if (valid) {
#pragma unroll
        for (int k = 0; k < LS; ++k) {
          hw = fma2(f[k], hw, bb[k]);
          if (full || t0 + warp * LS + k < T_) store_pair(op + (size_t)k * d, mul2(gg[k], hw));
        }
      }
    } else {
      // 1. gates and this warp's composed map
      float f[LS][CPL], bb[LS][CPL], gg[LS][CPL];
      float Aa[CPL], Bb[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        Aa[c] = 1.0f;
        Bb[c] = 0.0f;
      }
#pragma unroll
      for (int k = 0; k < LS; ++k) {
        const int tl = warp * LS + k;
        if (full || t0 + tl < T_) {
          float zf[CPL], zc[CPL], zg[CPL];
          LN::load(&tile[0][tl][lane * CPL], zf);
          LN::load(&tile[1][tl][lane * CPL], zc);
          LN::load(&tile[2][tl][lane * CPL], zg);
#pragma unroll
          for (int c = 0; c < CPL; ++c) gates(zf[c], zc[c], zg[c], f[k][c], bb[k][c], gg[k][c]);
        } else {   // past the end of the sequence: identity map
#pragma unroll
          for (int c = 0; c < CPL; ++c) {
            f[k][c] = 1.0f;
            bb[k][c] = 0.0f;
            gg[k][c] = 0.0f;
          }
        }
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          Bb[c] = fmaf(f[k][c], Bb[c], bb[k][c]);
          Aa[c] *= f[k][c];
        }
      }
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        sm.A[warp][c][lane] = Aa[c];
        sm.Bv[warp][c][lane] = Bb[c];
      }
      __syncthreads();
      // 2. as above, one channel per lane
      float hw[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        float hv = hin[c];
        for (int w = 0; w < warp; ++w) hv = fmaf(sm.A[w][c][lane], hv, sm.Bv[w][c][lane]);
        hw[c] = hv;
        if (warp == SW - 1) sm.hnext[c][lane] = fmaf(Aa[c], hv, Bb[c]);
      }
      // 3. replay this warp's steps and store o'
#pragma unroll
      for (int k = 0; k < LS; ++k) {
        float out[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          hw[c] = fmaf(f[k][c], hw[c], bb[k][c]);
          out[c] = gg[k][c] * hw[c];
        }
        if (valid && (full || t0 + warp * LS + k < T_)) LN::store(op + (size_t)k * d, out);
      }
    }
    __syncthreads();   // the stage and the warps' maps are free again; hnext is written
#pragma unroll
    for (int c = 0; c < CPL; ++c) hin[c] = sm.hnext[c][lane];
    if (threadIdx.x == 0 && j + nst < nchunk) {
      fence_proxy_async_smem();
      issue(j + nst);
    }
  }
  if (valid) LN::store(h + (size_t)b * d + ch, hin);
}

template <typename T, int CC>
cudaError_t launch_typed(const void* pre, int B, int T_, int d, float* h, void* o, int* status, long long wait_cycles,
                         int skip_chunk, cudaStream_t stream) {
  CUtensorMap map;
  const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  // box = one gate of one chunk (CC channels x TC steps); a stage holds 3 boxes
  if (!make_tma_2d(&map, pre, dt, (int)sizeof(T), (uint64_t)3 * d, (uint64_t)B * T_, CC, TC,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const int n_cb = ceil_div(d, CC);
  const size_t stage_bytes = sizeof(T) * 3 * TC * CC;
  const int nst = (int)std::max<size_t>(2, std::min<size_t>(kMaxStages, (192 * 1024) / stage_bytes));
  const size_t smem = 128 + tiles_offset<CC>() + nst * stage_bytes;
  auto kern = mlgru_scan_kernel<T, CC>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(B * n_cb), dim3(kThreads), smem, stream, map, B, T_, d, n_cb, nst, h,
                    static_cast<T*>(o), status, wait_cycles, skip_chunk);
}

}  // namespace

size_t mlgru_scan_ws_bytes(int, int, int) { return 256; }

cudaError_t launch_mlgru_scan(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, void* o, int* status,
                              cudaStream_t stream) {
  if (B == 0 || T == 0) return cudaSuccess;
  if (!tma_available()) return cudaErrorNotSupported;
  const long long wait = wait_limit_cycles();
  const int skip = test_hook("MMF_SCAN_SKIP_CHUNK");
  // 64 channels per CTA when that gives enough CTAs to cover the GPU, else 32
  const bool wide = (size_t)B * ceil_div(d, 64) >= (size_t)num_sms() * 3 / 4;
  if (dt == MMF_BF16)
    return wide ? launch_typed<bf16, 64>(pre, B, T, d, h, o, status, wait, skip, stream)
                : launch_typed<bf16, 32>(pre, B, T, d, h, o, status, wait, skip, stream);
  return wide ? launch_typed<float, 64>(pre, B, T, d, h, o, status, wait, skip, stream)
              : launch_typed<float, 32>(pre, B, T, d, h, o, status, wait, skip, stream);
}

}  // namespace mmf
