// One decode step (T = 1) of a whole MatMul-free block in one kernel launch
// (sm_100a): the f|c|g projections with the MLGRU step, the o projection with
// its residual, gate|up with the SiLU gate, and the down projection with its
// residual, separated by grid-wide barriers instead of kernel boundaries.
//
// "MatMul-free language models" (DataCamp blog), sections "Replacing MatMul
// with ternary operations" and "Core components: MLGRU and GLU"; the hysenlabs
// review, sections "FusedBitLinear" and "HGRN attention": every projection is
// a FusedBitLinear (RMSNorm, per-token absmax int8 codes, ternary accumulate,
// rescale); the token mixer is f = sigmoid, c = SiLU, g = sigmoid over the
// projections, h = f h + (1 - f) c, o' = g h, then the o projection; the
// channel mixer is SiLU(gate) * up, then the down projection.
//
// Why one kernel: at decode sizes each projection streams a few MB of packed
// weights, which HBM delivers in about a microsecond, while a dependent kernel
// boundary costs several. Here the four stages of a layer meet at three grid
// barriers, and every CTA copies the next stage's weight slice into shared
// memory (cp.async) as soon as its current MMA is done, so the weight stream
// overlaps the epilogue, the barrier and the next stage's row work.
//
// Launch: cooperative (every CTA resident; one per SM), 512 threads. Per stage
// a CTA owns the 16-row weight tiles b, b + G, b + 2G, ... of that stage's
// projection (G CTAs). Each CTA copies the stage's M <= 8 input rows into
// shared memory (all copies in flight at once) and quantises them there, in
// place (one warp per row, the same row routine and fp32 steps as the
// standalone quantiser, so the codes are the same); then its 16 warps take
// (tile, 256-column segment) pairs and accumulate with mma.sync m16n8k32 (u8
// codes w + 1 against s8 activations, the code sum subtracted afterwards),
// exactly as the separate decode contraction does; partial sums meet in
// shared memory through integer atomics (exact in any order). The epilogues
// use the same fp32 steps as the separate kernels.
//
// Grid barrier: a counter and a generation word, 128 bytes apart (zero between
// launches). The last CTA to arrive resets the counter and advances the
// generation; the others poll the generation, for at most kBarrierCycles,
// after which they record status code 4 and leave the kernel (the state words
// must then be reset before the next launch).
#include "kernels.cuh"
#include "quant_row.cuh"

namespace mmf {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr uint32_t kLow2 = 0x03030303u;
constexpr long long kBarrierCycles = 4000000000LL;   // ~2 s at 2 GHz

__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t u4get(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Activation-dtype element read through L2 (written by other CTAs of this grid).
__device__ __forceinline__ float ld_cg_f32(const float* p) { return __ldcg(p); }
__device__ __forceinline__ float ld_cg_f32(const bf16* p) { return __bfloat162float(__ldcg(p)); }

// Shared-memory pitch of one weight row in 16-byte units (row + 64 bytes, so
// the 8 rows a quarter-warp reads start in different banks). Token rows are
// staged K * esize + 16 bytes apart, and their codes overwrite the start of
// each row.
__host__ __device__ __forceinline__ int row_pitch4(int K) { return K / 64 + 4; }
__host__ __device__ __forceinline__ int token_pitch(int K, int esize) { return K * esize + 16; }

// Stage weight slice of CTA `b`: tiles b, b + G, ... ; tile ti, segment r, row
// i at 16-byte offset ((ti * R + r) * 16 + i) * pitch4. Rows past N read as 0.
__device__ void prefetch_stage(const DecodeStage& S, uint4* slot, int b, int G) {
  const int wpr4 = S.K / 64, pitch4 = row_pitch4(S.K);
  const int ntile = ceil_div(S.N, 16);
  const int ntl = b < ntile ? ceil_div(ntile - b, G) : 0;
  const int per_tile = S.nseg * 16 * wpr4;
  for (int idx = threadIdx.x; idx < ntl * per_tile; idx += kThreads) {
    const int ti = idx / per_tile, rem = idx - ti * per_tile;
    const int r = rem / (16 * wpr4), rem2 = rem - r * 16 * wpr4;
    const int row = rem2 / wpr4, c4 = rem2 - row * wpr4;
    const int n = (b + ti * G) * 16 + row;
    const bool ok = n < S.N;
    const uint32_t* src = ok ? S.w[r] + (size_t)n * (S.K / 16) + c4 * 4 : S.w[r];
    cp_async16(&slot[((ti * S.nseg + r) * 16 + row) * pitch4 + c4], src, ok);
  }
}

// Copy the stage's M token rows (K elements each, contiguous in global memory)
// into shared memory, rows token_pitch apart; all copies in flight at once.
template <typename T>
__device__ void stage_rows(const T* rows, int M, int K, uint8_t* rs) {
  const int nvec = (int)(K * sizeof(T) / 16), pitch = token_pitch(K, (int)sizeof(T));
  const uint4* src = reinterpret_cast<const uint4*>(rows);
  for (int i = threadIdx.x; i < M * nvec; i += kThreads) {
    const int m = i / nvec, v = i - m * nvec;
    cp_async16(rs + (size_t)m * pitch + v * 16, src + i, true);
  }
  cp_async_commit();
}

// Quantise the staged rows in place: warps 0..M-1, one row each; the codes
// take the first K bytes of each row.
template <typename T>
__device__ void quant_rows(uint8_t* rs, int M, int K, const float* gain, float eps, float* s_sm, int* qsum_sm) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= M) return;
  const int nvec = (int)(K * sizeof(T) / 16);
  uint8_t* row = rs + (size_t)warp * token_pitch(K, (int)sizeof(T));
  const uint4* xr = reinterpret_cast<const uint4*>(row);
  int8_t* qr = reinterpret_cast<int8_t*>(row);
  const RowCode rc = gain != nullptr ? quant_row<T, true, false, true>(xr, nvec, K, gain, eps, qr, lane)
                                     : quant_row<T, false, false, true>(xr, nvec, K, nullptr, eps, qr, lane);
  if (lane == 0) {
    s_sm[warp] = rc.scale;
    qsum_sm[warp] = rc.qsum;
  }
}

// Accumulators of this CTA's tiles of one stage into red[ti][r][row][token].
template <int R>
__device__ void stage_mma(const DecodeStage& S, const uint4* slot, const int8_t* qs, int qpitch, int M, int ntl,
                          int (*red)[3][16][8]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int K = S.K, wpr = K / 16, nkseg = ceil_div(K, 256);
  const int pitch4 = row_pitch4(K);
  for (int item = warp; item < ntl * nkseg; item += kWarps) {
    const int ti = item / nkseg, seg = item - ti * nkseg;
    const int w0 = seg * 16 + 4 * t;   // first packed word of this lane
    const bool in = w0 < wpr;          // wpr % 4 == 0: a 16-byte group is all in or all out
    uint4 wa[R], wb[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint4* base = slot + (size_t)((ti * R + r) * 16) * pitch4 + (w0 >> 2);
      wa[r] = in ? base[(size_t)g * pitch4] : make_uint4(0u, 0u, 0u, 0u);
      wb[r] = in ? base[(size_t)(g + 8) * pitch4] : make_uint4(0u, 0u, 0u, 0u);
    }
    uint4 act[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const bool ok = (g < M) && (w0 + u < wpr);
      act[u] = ok ? *reinterpret_cast<const uint4*>(qs + (size_t)g * qpitch + (w0 + u) * 16)
                  : make_uint4(0u, 0u, 0u, 0u);
    }
    int acc[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][e] = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int u = i >> 1, sub = (i & 1) * 2;
      const uint32_t b0 = u4get(act[u], sub), b1 = u4get(act[u], sub + 1);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t wg = u4get(wa[r], u), wg8 = u4get(wb[r], u);
        mma_u8s8(acc[r], (wg >> (2 * sub)) & kLow2, (wg8 >> (2 * sub)) & kLow2, (wg >> (2 * sub + 2)) & kLow2,
                 (wg8 >> (2 * sub + 2)) & kLow2, b0, b1);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      atomicAdd(&red[ti][r][g][2 * t], acc[r][0]);
      atomicAdd(&red[ti][r][g][2 * t + 1], acc[r][1]);
      atomicAdd(&red[ti][r][g + 8][2 * t], acc[r][2]);
      atomicAdd(&red[ti][r][g + 8][2 * t + 1], acc[r][3]);
    }
  }
}

// Grid-wide barrier (see the file comment). Returns false when the wait gave up.
__device__ bool grid_barrier(unsigned* bar, int* status, int* ok_sm) {
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile unsigned* gen = bar + 32;   // its own 128-byte line: polls do not queue behind the arrivals
    const unsigned g0 = *gen;
    __threadfence();
    bool ok = true;
    if (atomicAdd(bar, 1u) == gridDim.x - 1) {
      atomicExch(bar, 0u);
      __threadfence();
      atomicAdd(bar + 32, 1u);
    } else {
      const long long t0 = clock64();
      while (*gen == g0) {
        __nanosleep(32);
        if (clock64() - t0 > kBarrierCycles) {
          if (status) atomicExch(status, 4);
          ok = false;
          break;
        }
      }
    }
    __threadfence();
    *ok_sm = ok;
  }
  __syncthreads();
  return *ok_sm != 0;
}

// Stage P of the block (0: f|c|g + MLGRU step, 1: o + block input, 2: gate|up
// + SiLU gate, 3: down + token-mixer output) for this CTA. Its weight slice is
// already on the way into `slot`; once its MMA is done the slot takes stage
// P + 1's slice.
template <typename T, int P>
__device__ __forceinline__ void run_stage(const DecodeBlockArgs& a, uint4* slot, uint8_t* rs, int (*red)[3][16][8],
                                          float* s_sm, int* qsum_sm) {
  constexpr int R = P == 0 ? 3 : (P == 2 ? 2 : 1);
  const DecodeStage& S = a.st[P];
  const int b = blockIdx.x, G = gridDim.x, M = a.M;
  for (int i = threadIdx.x; i < kDecodeMaxTiles * 3 * 16 * 8; i += kThreads) (&red[0][0][0][0])[i] = 0;
  const void* in = P == 0 ? a.x : (P == 1 ? a.og : (P == 2 ? a.y1 : a.p));
  stage_rows<T>(static_cast<const T*>(in), M, S.K, rs);
  asm volatile("cp.async.wait_group 0;" ::: "memory");   // the rows and this stage's weight slice
  __syncthreads();
  quant_rows<T>(rs, M, S.K, S.gain, a.eps, s_sm, qsum_sm);
  __syncthreads();

  const int ntile = ceil_div(S.N, 16);
  const int ntl = b < ntile ? ceil_div(ntile - b, G) : 0;
  stage_mma<R>(S, slot, reinterpret_cast<const int8_t*>(rs), token_pitch(S.K, (int)sizeof(T)), M, ntl, red);
  __syncthreads();
  if constexpr (P < 3) {   // the slot is free: next stage's slice, behind the epilogue and the barrier
    prefetch_stage(a.st[P + 1], slot, b, G);
    cp_async_commit();
  }

  // epilogue: thread -> (tile, token, row), rows fastest so stores coalesce
  for (int idx = threadIdx.x; idx < ntl * 16 * M; idx += kThreads) {
    const int ti = idx / (16 * M), rem = idx - ti * 16 * M;
    const int m = rem >> 4, row = rem & 15;
    const int n = (b + ti * G) * 16 + row;
    if (n >= S.N) continue;
    const float s = s_sm[m];
    const int qsum = qsum_sm[m];
    if constexpr (P == 0) {   // f, c, g pre-activations -> one MLGRU step; h in place, o'
      float pre[3];
#pragma unroll
      for (int r = 0; r < 3; ++r) {
        float v = rescale_acc(red[ti][r][row][m] - qsum, *S.gamma[r], s);
        if (S.bias[r] != nullptr) v += S.bias[r][n];
        pre[r] = round_to<T>(v);   // the pre-activations are a storage point
      }
      float* hp = a.h + (size_t)m * a.d + n;
      float hn = *hp;
      const float og = mlgru_step(pre[0], pre[1], pre[2], hn);
      *hp = hn;
      static_cast<T*>(a.og)[(size_t)m * a.d + n] = from_f32<T>(og);
    } else if constexpr (P == 2) {   // gate, up -> SiLU(gate) * up
      float uv[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float v = rescale_acc(red[ti][r][row][m] - qsum, *S.gamma[r], s);
        if (S.bias[r] != nullptr) v += S.bias[r][n];
        uv[r] = v;
      }
      static_cast<T*>(a.p)[(size_t)m * a.I + n] = from_f32<T>(siluf_(uv[0]) * uv[1]);
    } else {   // o (+ block input, written before this launch) or down (+ y1, written by this grid)
      float v = rescale_acc(red[ti][0][row][m] - qsum, *S.gamma[0], s);
      if (S.bias[0] != nullptr) v += S.bias[0][n];
      if constexpr (P == 1) {
        v += to_f32(static_cast<const T*>(a.x)[(size_t)m * a.d + n]);
        static_cast<T*>(a.y1)[(size_t)m * a.d + n] = from_f32<T>(v);
      } else {
        v += ld_cg_f32(static_cast<const T*>(a.y1) + (size_t)m * a.d + n);
        static_cast<T*>(a.y)[(size_t)m * a.d + n] = from_f32<T>(v);
      }
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) decode_block_kernel(DecodeBlockArgs a) {
  extern __shared__ uint4 dsm[];   // weight slot [slot_bytes], then token rows / codes [M][token_pitch]
  __shared__ int red[kDecodeMaxTiles][3][16][8];
  __shared__ float s_sm[8];
  __shared__ int qsum_sm[8];
  __shared__ int ok_sm;
  uint4* slot = dsm;
  uint8_t* rs = reinterpret_cast<uint8_t*>(dsm + a.slot_bytes / 16);

  prefetch_stage(a.st[0], slot, blockIdx.x, gridDim.x);
  cp_async_commit();
  // after a barrier that gave up: no copy may land once the CTA is gone
  run_stage<T, 0>(a, slot, rs, red, s_sm, qsum_sm);
  if (!grid_barrier(a.bar, a.status, &ok_sm)) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    return;
  }
  run_stage<T, 1>(a, slot, rs, red, s_sm, qsum_sm);
  if (!grid_barrier(a.bar, a.status, &ok_sm)) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    return;
  }
  run_stage<T, 2>(a, slot, rs, red, s_sm, qsum_sm);
  if (!grid_barrier(a.bar, a.status, &ok_sm)) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    return;
  }
  run_stage<T, 3>(a, slot, rs, red, s_sm, qsum_sm);
}

// Bytes of one weight slot: the largest slice any stage gives one CTA.
size_t slot_bytes_for(const DecodeBlockArgs& a, int G) {
  size_t best = 0;
  for (int p = 0; p < 4; ++p) {
    const DecodeStage& S = a.st[p];
    const size_t tiles = (size_t)ceil_div(ceil_div(S.N, 16), G);
    best = std::max(best, tiles * S.nseg * 16 * (size_t)row_pitch4(S.K) * 16);
  }
  return best;
}

size_t smem_bytes_for(const DecodeBlockArgs& a, int G, int esize) {
  return slot_bytes_for(a, G) + (size_t)a.M * token_pitch(std::max(a.d, a.I), esize);
}

constexpr size_t kDecodeSmemLimit = 200 * 1024;   // dynamic part; the static part is ~6.3 KB

}  // namespace

bool decode_block_supported(const DecodeBlockArgs& a, mmf_dtype dt) {
  if (a.M < 1 || a.M > 8 || a.d % 64 != 0 || a.I % 64 != 0 || a.d < 64 || a.I < 64) return false;
  const int G = num_sms();
  if (G < 1) return false;
  for (int p = 0; p < 4; ++p) {
    const DecodeStage& S = a.st[p];
    if (S.K % 64 != 0 || S.N < 1) return false;
    if (ceil_div(ceil_div(S.N, 16), G) > kDecodeMaxTiles) return false;
  }
  return smem_bytes_for(a, G, (dt == MMF_BF16 ? 2 : 4)) <= kDecodeSmemLimit;
}

cudaError_t launch_decode_block(DecodeBlockArgs a, mmf_dtype dt, cudaStream_t stream) {
  const int G = num_sms();
  a.slot_bytes = (int)slot_bytes_for(a, G);
  const size_t smem = smem_bytes_for(a, G, (dt == MMF_BF16 ? 2 : 4));
  auto kern = dt == MMF_BF16 ? decode_block_kernel<bf16> : decode_block_kernel<float>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace mmf
