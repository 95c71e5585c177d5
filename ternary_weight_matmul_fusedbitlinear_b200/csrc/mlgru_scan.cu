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
// Work item = 32 channels of one sequence x one chunk of 256 steps; items are
// independent CTAs, so a sequence's chunks run in parallel:
//   1. TMA brings the item's f~, c~, g~ tile (3 x 256 x 32) into shared memory
//      as four 64-step parts with one barrier each.
//   2. Warp w (lane = channel) waits only for the part holding its steps
//      [16w, 16w+16), computes their gates, keeps f and b in registers and
//      composes its 16 steps into one map.
//   3. Warp 0 takes the state entering the chunk - h_0 for the first chunk,
//      otherwise the state the previous chunk of the same channels publishes -
//      folds the 16 warp maps over it, records each warp's entering state, and
//      publishes the state leaving the chunk (value, then a release flag).
//   4. Every warp replays its 16 steps from its entering state and writes o'.
// Forward progress: an item takes a ticket from a global counter and derives
// its coordinates from it, chunk-major, so the item it waits on (same
// channels, previous chunk) took an earlier ticket and is already running or
// done. The wait is bounded: on timeout the kernel records status 2 and
// continues with a zero state (the results are then invalid and mmf_check
// reports MMF_ERR_TIMEOUT); nothing spins forever.
#include "kernels.cuh"
#include "tma.cuh"

namespace mmf {

namespace {

constexpr int CC = 32;          // channels per item (one per lane)
constexpr int TC = 256;         // steps per chunk
constexpr int SW = 16;          // warps per CTA
constexpr int LS = TC / SW;     // steps per warp
constexpr int NPART = 4;        // TMA parts per chunk
constexpr int PS = TC / NPART;  // steps per part
constexpr int kThreads = SW * 32;

__device__ __forceinline__ float sigmoid_fast(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }

template <typename T>
struct ScanSmem {
  T tile[3][TC][CC];              // [gate f,c,g][step][channel]
  float A[SW][CC];                // composed multiplier of each warp's steps
  float Bv[SW][CC];               // composed offset
  float start[SW][CC];            // state entering each warp's steps
  uint64_t full[NPART];
  int ticket;
  int abort_flag;
};

// Per-launch scratch: ticket counter, one flag per item, then one 32-channel
// state per item (the state leaving that chunk).
struct ScanWs {
  int* ticket;
  int* flags;
  float* carry;
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2) mlgru_scan_kernel(const __grid_constant__ CUtensorMap map, int B, int T_,
                                                              int d, int n_cb, int nchunk, float* __restrict__ h,
                                                              T* __restrict__ o, ScanWs ws, int* status) {
  extern __shared__ uint8_t smem_raw[];
  ScanSmem<T>& sm = *reinterpret_cast<ScanSmem<T>*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kPartBytes = 3u * PS * CC * sizeof(T);

  if (threadIdx.x == 0) {
    sm.ticket = atomicAdd(ws.ticket, 1);
    for (int q = 0; q < NPART; ++q) mbar_init(&sm.full[q], 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int item = sm.ticket;                         // chunk-major order
  const int per_chunk = B * n_cb;
  const int j = item / per_chunk, rem = item - j * per_chunk;
  const int b = rem / n_cb, cb = rem - b * n_cb;
  const int c0 = cb * CC, ch = c0 + lane;
  const bool valid = ch < d;
  const int t0 = j * TC;
  const int row0 = b * T_ + t0;
  if (threadIdx.x == 0) {
    for (int q = 0; q < NPART; ++q) {
      if (t0 + q * PS >= T_) break;                     // nothing of this part is in the sequence
      mbar_arrive_expect_tx(&sm.full[q], kPartBytes);
      for (int g = 0; g < 3; ++g)
        tma_load_2d(&sm.tile[g][q * PS][0], &map, g * d + c0, row0 + q * PS, &sm.full[q]);
    }
  }
  const int part = (warp * LS) / PS;
  const bool need = t0 + part * PS < T_;
  const bool got = need ? mbar_wait(&sm.full[part], 0, &sm.abort_flag, status) : true;
  if (__syncthreads_or(!got)) {
    if (threadIdx.x == 0) {
      for (int q = 0; q < NPART && t0 + q * PS < T_; ++q)
        mbar_wait(&sm.full[q], 0, &sm.abort_flag, nullptr);   // let the copies land
      st_release(ws.flags + item, 1);                          // successors must not wait on this item
    }
    return;
  }

  // 2. gates and this warp's composed map
  float f[LS], bb[LS];
  float Aa = 1.0f, Bb = 0.0f;
#pragma unroll
  for (int k = 0; k < LS; ++k) {
    const int tl = warp * LS + k;
    if (t0 + tl < T_) {
      const float fv = sigmoid_fast(to_f32(sm.tile[0][tl][lane]));
      const float cz = to_f32(sm.tile[1][tl][lane]);
      f[k] = fv;
      bb[k] = (1.0f - fv) * (cz * sigmoid_fast(cz));
    } else {   // past the end of the sequence: identity map
      f[k] = 1.0f;
      bb[k] = 0.0f;
    }
    Bb = f[k] * Bb + bb[k];
    Aa *= f[k];
  }
  sm.A[warp][lane] = Aa;
  sm.Bv[warp][lane] = Bb;
  __syncthreads();

  // 3. state entering the chunk, per-warp entering states, publish the leaving state
  if (warp == 0) {
    const size_t slot = (size_t)j * per_chunk + rem;          // this item
    float hv = 0.0f;
    if (j == 0) {
      hv = valid ? h[(size_t)b * d + ch] : 0.0f;
    } else {
      const size_t prev = slot - per_chunk;                    // same channels, previous chunk
      int ok = 1;
      if (lane == 0) {
        const long long t_start = clock64();
        while (ld_acquire(ws.flags + prev) == 0) {
          if (clock64() - t_start > kWaitCycles) {
            ok = 0;
            atomicExch(status, 2);
            break;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok && ld_acquire(ws.flags + prev) != 0) hv = __ldcg(ws.carry + prev * CC + lane);
    }
#pragma unroll
    for (int w = 0; w < SW; ++w) {
      sm.start[w][lane] = hv;
      hv = sm.A[w][lane] * hv + sm.Bv[w][lane];
    }
    ws.carry[slot * CC + lane] = hv;
    __syncwarp();
    if (lane == 0) {
      __threadfence();
      st_release(ws.flags + slot, 1);
    }
    if (j == nchunk - 1 && valid) h[(size_t)b * d + ch] = hv;
  }
  __syncthreads();

  // 4. replay this warp's steps
  float hv = sm.start[warp][lane];
  T* op = o + ((size_t)row0 + warp * LS) * d + ch;
#pragma unroll
  for (int k = 0; k < LS; ++k) {
    const int tl = warp * LS + k;
    hv = f[k] * hv + bb[k];
    if (valid && t0 + tl < T_) {
      const float gv = sigmoid_fast(to_f32(sm.tile[2][tl][lane]));
      op[(size_t)k * d] = from_f32<T>(gv * hv);
    }
  }
}

template <typename T>
cudaError_t launch_typed(const void* pre, int B, int T_, int d, float* h, void* o, void* ws, int* status,
                         cudaStream_t stream) {
  CUtensorMap map;
  const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  // box = one part (PS steps x CC channels of one gate): each part load fills exactly
  // tile[g][q*PS .. q*PS+PS) and its barrier expects 3 * PS * CC elements
  if (!make_tma_2d(&map, pre, dt, (int)sizeof(T), (uint64_t)3 * d, (uint64_t)B * T_, CC, PS,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const int n_cb = ceil_div(d, CC), nchunk = ceil_div(T_, TC);
  const int items = nchunk * B * n_cb;
  char* base = static_cast<char*>(ws);
  ScanWs w;
  w.ticket = reinterpret_cast<int*>(base);
  w.flags = w.ticket + 1;
  w.carry = reinterpret_cast<float*>(base + (sizeof(int) * (size_t)(items + 1) + 255) / 256 * 256);
  cudaError_t e = cudaMemsetAsync(base, 0, sizeof(int) * (size_t)(items + 1), stream);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(ScanSmem<T>) + 128;
  auto kern = mlgru_scan_kernel<T>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<items, kThreads, smem, stream>>>(map, B, T_, d, n_cb, nchunk, h, static_cast<T*>(o), w, status);
  return cudaGetLastError();
}

}  // namespace

size_t mlgru_scan_ws_bytes(int B, int T, int d) {
  if (B <= 0 || T <= 0 || d <= 0) return 256;
  const size_t items = (size_t)ceil_div(T, TC) * B * ceil_div(d, CC);
  return (sizeof(int) * (items + 1) + 255) / 256 * 256 + sizeof(float) * items * CC;
}

cudaError_t launch_mlgru_scan(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, void* o, void* ws,
                              int* status, cudaStream_t stream) {
  if (B == 0 || T == 0) return cudaSuccess;
  if (!tma_available()) return cudaErrorNotSupported;
  return dt == MMF_BF16 ? launch_typed<bf16>(pre, B, T, d, h, o, ws, status, stream)
                        : launch_typed<float>(pre, B, T, d, h, o, ws, status, stream);
}

}  // namespace mmf
