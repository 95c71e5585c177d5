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
// Parallel form. Each step is the affine map h -> f h + b with b = (1 - f) c,
// and affine maps compose: (f2, b2) o (f1, b1) = (f2 f1, f2 b1 + b2).
// Work item = 64 channels of one sequence x one chunk of 128 steps (lane l
// owns channels 2l and 2l+1). Persistent CTAs take items from a global ticket
// counter, chunk-major, and keep the next item's tile in flight (TMA, 2-deep
// ring) while they compute the current one:
//   1. Warp w computes the gates of steps [16w, 16w+16), keeps f and b in
//      registers and composes its 16 steps into one map.
//   2. Every warp folds the maps of the warps before it (its entering map);
//      warp 0 folds all of them into the item's map and publishes it at once
//      (the "aggregate"), before it knows the state entering the chunk.
//   3. Warp 0 finds the entering state by looking back over the same
//      channels' previous chunks: a chunk that has published its leaving
//      state ends the walk, one that has published only its aggregate is
//      composed in and the walk goes one chunk further back. Chunk 0 starts
//      from h_0. It then publishes the leaving state.
//   4. Every warp replays its 16 steps from its entering state and writes o'.
// Because aggregates do not wait on anything, no chunk waits for a chain of
// predecessors to finish one after another. Publication needs no fence: each
// lane publishes its two channels' values as one 64-bit word, and the scratch
// is filled with an all-ones pattern (a NaN that arithmetic never produces)
// before the launch, so a word that is not all-ones in either half is ready.
// Forward progress: every wait is on an item with a smaller ticket; a CTA
// works on its tickets in increasing order, so the smallest unfinished ticket
// always belongs to a CTA that is working on it and whose predecessors are
// done. Waits are still bounded: on timeout the kernel records status 2 and
// continues with a zero state (results invalid; mmf_check reports
// MMF_ERR_TIMEOUT); nothing spins forever.
#include "kernels.cuh"
#include "tma.cuh"

namespace mmf {

namespace {

constexpr int CC = 64;          // channels per item
constexpr int TC = 128;         // steps per item
constexpr int SW = 8;           // warps per CTA
constexpr int LS = TC / SW;     // steps per warp
constexpr int NST = 2;          // item ring depth
constexpr int kThreads = SW * 32;
constexpr int kWsPerItem = 3 * CC;   // floats: aggregate multiplier, aggregate offset, leaving state
constexpr uint32_t kUnset = 0xffffffffu;

template <typename T>
struct ScanSmem {
  T tile[NST][3][TC][CC];         // [stage][gate f,c,g][step][channel]
  float2 A[SW][32];               // composed multiplier of each warp's steps (per lane: 2 channels)
  float2 Bv[SW][32];              // composed offset
  float2 hin[32];                 // state entering the item
  uint64_t full[NST];
  int tk[NST];                    // ticket held by each stage
  int abort_flag;
};

// Per-launch scratch, filled with all-ones bytes before the launch: ticket
// counter (starts at -1), then per item three fields of 32 lane words (float2
// each): aggregate multiplier, aggregate offset, leaving state.
struct ScanWs {
  int* ticket;
  float2* rec;
};

__device__ __forceinline__ float2 ld_word(const float2* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return make_float2(__uint_as_float((uint32_t)v), __uint_as_float((uint32_t)(v >> 32)));
}
__device__ __forceinline__ void st_word(float2* p, float2 v) {
  const uint64_t w = (uint64_t)__float_as_uint(v.x) | ((uint64_t)__float_as_uint(v.y) << 32);
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ bool is_set(float2 v) {
  return __float_as_uint(v.x) != kUnset && __float_as_uint(v.y) != kUnset;
}

__device__ __forceinline__ float2 load2(const bf16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ float2 load2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ void store2(bf16* p, float2 v) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v.x, v.y);
}
__device__ __forceinline__ void store2(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }

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
constexpr float kMaxExp2 = 40.0f * kLog2e;   // e^-z capped at e^40

// 1 / (1 + e^-z); e^-z overflows to +inf for z < -88 and the reciprocal gives 0
__device__ __forceinline__ float sigmoid_fast(float z) { return rcp_approx(1.0f + ex2_approx(-z * kLog2e)); }

// f = sigmoid(zf) and b = (1 - f) SiLU(zc) with one reciprocal for both
// logistic terms: 1/(1+e^-zf) = (1+e^-zc) r and 1/(1+e^-zc) = (1+e^-zf) r with
// r = 1/((1+e^-zf)(1+e^-zc)). The exponents are capped at 40 so the product
// stays finite; below -40 the logistic is under 5e-18 and the cap moves it by
// less than that.
__device__ __forceinline__ void gate_fb(float zf, float zc, float& f, float& b) {
  const float pf = 1.0f + ex2_approx(fminf(-zf * kLog2e, kMaxExp2));
  const float pc = 1.0f + ex2_approx(fminf(-zc * kLog2e, kMaxExp2));
  const float r = rcp_approx(pf * pc);
  f = pc * r;
  b = (1.0f - f) * (zc * (pf * r));
}

__device__ __forceinline__ float2 fma2(float2 a, float2 x, float2 b) {
  return make_float2(fmaf(a.x, x.x, b.x), fmaf(a.y, x.y, b.y));
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return make_float2(a.x * b.x, a.y * b.y); }

// Bounded wait for a stage's copies after an abort (ignores the abort flag).
__device__ void drain_stage(uint64_t* bar, uint32_t parity) {
  const long long t_start = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t_start < kWaitCycles / 10) {
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, sizeof(T) == 2 ? 2 : 1)
    mlgru_scan_kernel(const __grid_constant__ CUtensorMap map, int B, int T_, int d, int n_cb, int nchunk,
                      float* __restrict__ h, T* __restrict__ o, ScanWs ws, int* status) {
  extern __shared__ uint8_t smem_raw[];
  ScanSmem<T>& sm = *reinterpret_cast<ScanSmem<T>*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_chunk = B * n_cb;
  const int items = nchunk * per_chunk;
  constexpr uint32_t kItemBytes = 3u * TC * CC * sizeof(T);

  // thread 0: start the copies of ticket t into stage s (an out-of-range
  // ticket completes the stage's phase with no data)
  auto issue = [&](int s, int t) {
    sm.tk[s] = t;
    if (t < items) {
      const int j = t / per_chunk, rem = t - j * per_chunk;
      const int b = rem / n_cb, cb = rem - b * n_cb;
      mbar_arrive_expect_tx(&sm.full[s], kItemBytes);
      for (int g = 0; g < 3; ++g)
        tma_load_2d(&sm.tile[s][g][0][0], &map, g * d + cb * CC, b * T_ + j * TC, &sm.full[s]);
    } else {
      mbar_arrive(&sm.full[s]);
    }
  };

  pdl_trigger();
  pdl_wait();   // the pre-activations are the previous kernel's output
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) mbar_init(&sm.full[s], 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int s = 0; s < NST; ++s) issue(s, atomicAdd(ws.ticket, 1) + 1);
  }
  __syncthreads();

  for (int it = 0;; ++it) {
    const int s = it % NST;
    const uint32_t parity = (uint32_t)(it / NST) & 1u;
    const bool got = mbar_wait(&sm.full[s], parity, &sm.abort_flag, status);
    if (__syncthreads_or(!got)) {
      // give up: let successors of the held items go on (zero leaving state),
      // after the copies in flight have landed or a bounded wait has passed
      if (warp == 0) {
        for (int q = 0; q < NST; ++q) {
          const int sq = (it + q) % NST;
          const int t = sm.tk[sq];
          if (t >= items) continue;
          if (lane == 0) drain_stage(&sm.full[sq], (uint32_t)((it + q) / NST) & 1u);
          __syncwarp();
          st_word(ws.rec + ((size_t)t * 3 + 2) * 32 + lane, make_float2(0.0f, 0.0f));
        }
      }
      return;
    }
    const int item = sm.tk[s];
    if (item >= items) break;   // tickets rise, so every later stage is out of range too
    int next_ticket = 0;
    if (threadIdx.x == 0) next_ticket = atomicAdd(ws.ticket, 1) + 1;   // used at the end of the item

    const int j = item / per_chunk, rem = item - j * per_chunk;
    const int b = rem / n_cb, cb = rem - b * n_cb;
    const int ch = cb * CC + 2 * lane;
    const bool valid = ch < d;          // d is even, so ch + 1 < d too
    const int t0 = j * TC;
    const int row0 = b * T_ + t0;
    const T(*tile)[TC][CC] = sm.tile[s];

    // 1. gates and this warp's composed map
    float2 f[LS], bb[LS];
    float2 Aa = make_float2(1.0f, 1.0f), Bb = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < LS; ++k) {
      const int tl = warp * LS + k;
      if (t0 + tl < T_) {
        const float2 zf = load2(&tile[0][tl][2 * lane]);
        const float2 zc = load2(&tile[1][tl][2 * lane]);
        gate_fb(zf.x, zc.x, f[k].x, bb[k].x);
        gate_fb(zf.y, zc.y, f[k].y, bb[k].y);
      } else {   // past the end of the sequence: identity map
        f[k] = make_float2(1.0f, 1.0f);
        bb[k] = make_float2(0.0f, 0.0f);
      }
      Bb = fma2(f[k], Bb, bb[k]);
      Aa = mul2(Aa, f[k]);
    }
    sm.A[warp][lane] = Aa;
    sm.Bv[warp][lane] = Bb;
    __syncthreads();

    // 2. entering map of this warp (warps before it), and the item's map (warp 0)
    float2 pa = make_float2(1.0f, 1.0f), pb = make_float2(0.0f, 0.0f);
    for (int w = 0; w < warp; ++w) {
      const float2 a = sm.A[w][lane], c = sm.Bv[w][lane];
      pb = fma2(a, pb, c);
      pa = mul2(a, pa);
    }

    // 3. state entering the item; publish the aggregate, then the leaving state
    if (warp == 0) {
      float2 ta = make_float2(1.0f, 1.0f), tb = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int w = 0; w < SW; ++w) {
        const float2 a = sm.A[w][lane], c = sm.Bv[w][lane];
        tb = fma2(a, tb, c);
        ta = mul2(a, ta);
      }
      float2* mine = ws.rec + (size_t)item * 3 * 32 + lane;
      float2 hv = make_float2(0.0f, 0.0f);
      if (j == 0) {
        if (valid) hv = *reinterpret_cast<const float2*>(h + (size_t)b * d + ch);
      } else {
        st_word(mine, ta);
        st_word(mine + 32, tb);
        // look back: h_in = acc_a * (state leaving chunk p) + acc_b
        float2 acc_a = make_float2(1.0f, 1.0f), acc_b = make_float2(0.0f, 0.0f);
        int p = item - per_chunk;
        const long long t_start = clock64();
        while (true) {
          const float2* theirs = ws.rec + (size_t)p * 3 * 32 + lane;
          const float2 hp = ld_word(theirs + 64);
          const float2 a = ld_word(theirs), c = ld_word(theirs + 32);
          if (is_set(hp)) {
            hv = fma2(acc_a, hp, acc_b);
            break;
          }
          if (is_set(a) && is_set(c)) {              // aggregate only: compose it, look one chunk further
            acc_b = fma2(acc_a, c, acc_b);
            acc_a = mul2(acc_a, a);
            p -= per_chunk;                          // chunk 0 always publishes its leaving state
            continue;
          }
          if (clock64() - t_start > kWaitCycles) {   // give up: continue from zero (reported)
            atomicExch(status, 2);
            break;
          }
        }
      }
      sm.hin[lane] = hv;
      const float2 hout = fma2(ta, hv, tb);
      st_word(mine + 64, hout);
      if (j == nchunk - 1 && valid) *reinterpret_cast<float2*>(h + (size_t)b * d + ch) = hout;
    }
    __syncthreads();

    // 4. replay this warp's steps
    float2 hv = fma2(pa, sm.hin[lane], pb);
    T* op = o + ((size_t)row0 + warp * LS) * d + ch;
#pragma unroll
    for (int k = 0; k < LS; ++k) {
      const int tl = warp * LS + k;
      hv = fma2(f[k], hv, bb[k]);
      if (valid && t0 + tl < T_) {
        const float2 zg = load2(&tile[2][tl][2 * lane]);
        store2(op + (size_t)k * d, make_float2(sigmoid_fast(zg.x) * hv.x, sigmoid_fast(zg.y) * hv.y));
      }
    }
    __syncthreads();   // the stage is free again
    if (threadIdx.x == 0) issue(s, next_ticket);
  }
}

size_t ws_used_bytes(int B, int T_, int d) {
  const size_t items = (size_t)ceil_div(T_, TC) * B * ceil_div(d, CC);
  return 256 + sizeof(float) * items * kWsPerItem;
}

template <typename T>
cudaError_t launch_typed(const void* pre, int B, int T_, int d, float* h, void* o, void* ws, int* status,
                         cudaStream_t stream) {
  CUtensorMap map;
  const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  // box = one gate of one item (CC channels x TC steps); the stage barrier expects 3 boxes
  if (!make_tma_2d(&map, pre, dt, (int)sizeof(T), (uint64_t)3 * d, (uint64_t)B * T_, CC, TC,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const int n_cb = ceil_div(d, CC), nchunk = ceil_div(T_, TC);
  const int items = nchunk * B * n_cb;
  char* base = static_cast<char*>(ws);
  ScanWs w;
  w.ticket = reinterpret_cast<int*>(base);
  w.rec = reinterpret_cast<float2*>(base + 256);
  const size_t smem = sizeof(ScanSmem<T>) + 128;
  auto kern = mlgru_scan_kernel<T>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  const int grid = std::max(1, std::min(items, num_sms() * std::max(per_sm, 1)));
  return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, stream, map, B, T_, d, n_cb, nchunk, h,
                    static_cast<T*>(o), w, status);
}

}  // namespace

size_t mlgru_scan_ws_bytes(int B, int T, int d) {
  if (B <= 0 || T <= 0 || d <= 0) return 256;
  return ws_used_bytes(B, T, d);
}

cudaError_t reset_mlgru_scan_ws(void* ws, int B, int T, int d, cudaStream_t stream) {
  if (B <= 0 || T <= 0 || d <= 0) return cudaSuccess;
  return cudaMemsetAsync(ws, 0xff, ws_used_bytes(B, T, d), stream);
}

cudaError_t launch_mlgru_scan(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, void* o, void* ws,
                              int* status, cudaStream_t stream) {
  if (B == 0 || T == 0) return cudaSuccess;
  if (!tma_available()) return cudaErrorNotSupported;
  return dt == MMF_BF16 ? launch_typed<bf16>(pre, B, T, d, h, o, ws, status, stream)
                        : launch_typed<float>(pre, B, T, d, h, o, ws, status, stream);
}

}  // namespace mmf
