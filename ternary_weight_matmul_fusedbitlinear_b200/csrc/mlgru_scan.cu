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
// and affine maps compose: (f2, b2) o (f1, b1) = (f2 f1, f2 b1 + b2). A CTA
// owns 32 channels of one sequence and walks the sequence in tiles of 64
// steps, staged in shared memory by TMA (3-stage pipeline). Inside a tile,
// warp s takes steps [8s, 8s+8) for all 32 channels (lane = channel): it
// computes its gates once, keeps them in registers, composes its 8 steps into
// one map, publishes it, folds the maps of warps 0..s-1 into the tile's carry
// to get its starting state, then replays its 8 steps to produce o'. The carry
// out of the last warp seeds the next tile.
//
// Gates: the three logistic functions of a step share one reciprocal. With
// e_i = exp(-z_i) and D = (1+e_f)(1+e_c)(1+e_g), 1/(1+e_f) = (1+e_c)(1+e_g)/D
// and so on; the arguments are clamped to [-20, 20] first so D stays finite
// (sigmoid(20) rounds to 1 in fp32 and sigmoid(-20) = 2.1e-9 is below the
// output tolerance), which takes 3 exponentials and 1 reciprocal per step.
#include "kernels.cuh"
#include "tma.cuh"

namespace mmf {

namespace {

constexpr int CC = 32;          // channels per CTA (one per lane)
constexpr int TC = 64;          // steps per tile
constexpr int SW = 8;           // warps (sub-chunks) per CTA
constexpr int LS = TC / SW;     // steps per warp per tile
constexpr int STAGES = 3;
constexpr int kThreads = SW * 32;

// sigmoid of three arguments with one reciprocal (see the file comment)
__device__ __forceinline__ void sigmoid3(float zf, float zc, float zg, float& sf, float& sc, float& sg) {
  const float af = 1.0f + __expf(-fminf(fmaxf(zf, -20.0f), 20.0f));
  const float ac = 1.0f + __expf(-fminf(fmaxf(zc, -20.0f), 20.0f));
  const float ag = 1.0f + __expf(-fminf(fmaxf(zg, -20.0f), 20.0f));
  const float fc = af * ac;
  const float r = __fdividef(1.0f, fc * ag);
  sg = r * fc;
  const float rg = r * ag;
  sf = rg * ac;
  sc = rg * af;
}

template <typename T>
struct ScanSmem {
  T tile[STAGES][3][TC][CC];      // [stage][gate f,c,g][step][channel]
  float A[2][SW][CC];             // composed multiplier of each warp's steps (double-buffered by tile parity)
  float Bv[2][SW][CC];            // composed offset
  float carry[2][CC];             // state entering the tile
  uint64_t full[STAGES];
  int abort_flag;
};

template <typename T>
__global__ void __launch_bounds__(kThreads) mlgru_scan_kernel(const __grid_constant__ CUtensorMap map, int T_,
                                                              int d, int n_cb, float* __restrict__ h,
                                                              T* __restrict__ o, int* status) {
  extern __shared__ uint8_t smem_raw[];
  ScanSmem<T>& sm = *reinterpret_cast<ScanSmem<T>*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x / n_cb, cb = blockIdx.x % n_cb;
  const int c0 = cb * CC, ch = c0 + lane;
  const bool valid = ch < d;
  const int ntiles = ceil_div(T_, TC);
  const int row_base = b * T_;
  constexpr uint32_t kTileBytes = 3u * TC * CC * sizeof(T);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&sm.full[s], 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&map);
  }
  if (warp == 0) sm.carry[0][lane] = valid ? h[(size_t)b * d + ch] : 0.0f;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES && i < ntiles; ++i) {
      mbar_arrive_expect_tx(&sm.full[i], kTileBytes);
      for (int g = 0; g < 3; ++g) tma_load_2d(&sm.tile[i][g][0][0], &map, g * d + c0, row_base + i * TC, &sm.full[i]);
    }
  }

  int i = 0;
  for (; i < ntiles; ++i) {
    const int s = i % STAGES, par = i & 1;
    const bool got = mbar_wait(&sm.full[s], (i / STAGES) & 1, &sm.abort_flag, status);
    if (__syncthreads_or(!got)) break;
    const int t0 = i * TC + warp * LS;
    float f[LS], bb[LS], gg[LS];
    float Aa = 1.0f, Bb = 0.0f;
#pragma unroll
    for (int j = 0; j < LS; ++j) {
      const int tl = warp * LS + j;
      if (t0 + j < T_) {
        const float cz = to_f32(sm.tile[s][1][tl][lane]);
        float fv, sc, gv;
        sigmoid3(to_f32(sm.tile[s][0][tl][lane]), cz, to_f32(sm.tile[s][2][tl][lane]), fv, sc, gv);
        gg[j] = gv;
        f[j] = fv;
        bb[j] = (1.0f - fv) * (cz * sc);
      } else {   // past the end: identity map
        f[j] = 1.0f;
        bb[j] = 0.0f;
        gg[j] = 0.0f;
      }
      Bb = f[j] * Bb + bb[j];
      Aa *= f[j];
    }
    sm.A[par][warp][lane] = Aa;
    sm.Bv[par][warp][lane] = Bb;
    __syncthreads();   // maps published; every thread is done reading stage s
    if (threadIdx.x == 0 && i + STAGES < ntiles) {
      mbar_arrive_expect_tx(&sm.full[s], kTileBytes);
      for (int g = 0; g < 3; ++g)
        tma_load_2d(&sm.tile[s][g][0][0], &map, g * d + c0, row_base + (i + STAGES) * TC, &sm.full[s]);
    }
    float hv = sm.carry[par][lane];
    for (int w = 0; w < warp; ++w) hv = sm.A[par][w][lane] * hv + sm.Bv[par][w][lane];
    if (warp == SW - 1) sm.carry[par ^ 1][lane] = Aa * hv + Bb;
    T* op = o + ((size_t)row_base + t0) * d + ch;
#pragma unroll
    for (int j = 0; j < LS; ++j) {
      hv = f[j] * hv + bb[j];
      if (valid && t0 + j < T_) op[(size_t)j * d] = from_f32<T>(gg[j] * hv);
    }
  }
  __syncthreads();
  if (warp == SW - 1 && valid && i == ntiles) h[(size_t)b * d + ch] = sm.carry[ntiles & 1][lane];
  if (i < ntiles && threadIdx.x == 0) {
    // aborted: let the copies already issued land before shared memory is released
    for (int j = i; j < ntiles && j < i + STAGES; ++j)
      mbar_wait(&sm.full[j % STAGES], (j / STAGES) & 1, &sm.abort_flag, nullptr);
  }
}

template <typename T>
cudaError_t launch_typed(const void* pre, int B, int T_, int d, float* h, void* o, int* status, cudaStream_t stream) {
  CUtensorMap map;
  const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  if (!make_tma_2d(&map, pre, dt, (int)sizeof(T), (uint64_t)3 * d, (uint64_t)B * T_, CC, TC,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(ScanSmem<T>) + 128;
  auto kern = mlgru_scan_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n_cb = ceil_div(d, CC);
  kern<<<B * n_cb, kThreads, smem, stream>>>(map, T_, d, n_cb, h, static_cast<T*>(o), status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mlgru_scan(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, void* o, int* status,
                              cudaStream_t stream) {
  if (B == 0 || T == 0) return cudaSuccess;
  if (!tma_available()) return cudaErrorNotSupported;
  return dt == MMF_BF16 ? launch_typed<bf16>(pre, B, T, d, h, o, status, stream)
                        : launch_typed<float>(pre, B, T, d, h, o, status, stream);
}

}  // namespace mmf
