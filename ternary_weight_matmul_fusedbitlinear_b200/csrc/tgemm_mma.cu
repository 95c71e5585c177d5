// Packed-ternary x int8 contraction on the warp-level tensor-core MMA
// (mma.sync m16n8k32, u8 x s8 -> s32). Used for decode-sized token counts,
// where the kernel streams the 2-bit weights from HBM once.
//
// "MatMul-free language models" (DataCamp blog), section "Replacing MatMul
// with ternary operations": a product with a weight of -1, 0 or 1 is a
// negation, a drop or a copy, so acc[m, n] = sum_k q[m,k] * w[n,k] is exact
// integer add/subtract work. Here the stored code is w + 1 in {0,1,2}; the
// kernel multiplies the stored code as an unsigned byte and subtracts the
// per-token code sum afterwards: sum_k (w+1) q = acc + sum_k q.
//
// Launch: programmatic dependent launch. Before waiting on its predecessor a
// CTA copies its whole weight slice (16 rows x K of each segment) into shared
// memory with cp.async, so the weight stream overlaps the previous kernel; the
// activations are read only after pdl_wait().
//
// Fused quantisation (FQ): for decode-sized token counts every CTA can take the
// raw activations instead of int8 codes and quantise its (at most 16) token
// rows itself, one warp per row, with the same row routine and the same fp32
// steps as the standalone quantiser, so the codes are identical; one kernel per
// projection instead of two. The rows are first copied whole into shared
// memory (all copies in flight at once), so their latency is paid once.
//
// Work split: a CTA owns 16 output rows of each of its R weight segments and
// 8*NT tokens; its 8 warps split K into 256-column segments round-robin. Per
// 256-column segment a lane (group g, thread t) loads 16 bytes of packed codes
// for rows g and g+8 (64 columns) and the 64 activation bytes [64t, 64t+64) of
// its token; the column order inside the segment is permuted identically on
// both operands, which the sum does not see. Partial sums meet in shared
// memory through integer atomics (exact in any order), then the epilogue
// rescales and applies the mode.
#include "kernels.cuh"
#include "quant_row.cuh"

namespace mmf {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = 8;
constexpr uint32_t kLow2 = 0x03030303u;

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

// Load 4 consecutive 32-bit words starting at word index `w0` of a row with
// `nw` words; words at or beyond nw read as 0. One 16-byte load only when the
// rows are 16-byte aligned (nw % 4 == 0, so every row starts on a 16-byte
// boundary of the 16-byte aligned matrix) and all 4 words are in the row.
__device__ __forceinline__ uint4 load_words4(const uint32_t* row, int w0, int nw, bool row_ok) {
  uint4 r = make_uint4(0u, 0u, 0u, 0u);
  if (!row_ok) return r;
  if ((nw & 3) == 0 && w0 + 4 <= nw) return __ldg(reinterpret_cast<const uint4*>(row + w0));
  if (w0 + 0 < nw) r.x = __ldg(row + w0 + 0);
  if (w0 + 1 < nw) r.y = __ldg(row + w0 + 1);
  if (w0 + 2 < nw) r.z = __ldg(row + w0 + 2);
  if (w0 + 3 < nw) r.w = __ldg(row + w0 + 3);
  return r;
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(valid ? 16 : 0) : "memory");
}

// Shared-memory pitch of one weight row in 16-byte units: the row plus 64 bytes,
// so the 8 rows a quarter-warp reads start in different banks.
__host__ __device__ __forceinline__ int wsm_pitch4(int wpr) { return wpr / 4 + 4; }

// Shared-memory row pitch (bytes) of the fused-quantisation codes: 16 bytes
// more than a row, which spreads the 8 rows of a fragment load over the banks.
__host__ __device__ __forceinline__ int fq_pitch(int K) { return K + 16; }

// FQM: how the kernel gets its activation codes. 0: from the standalone
// quantiser (a.q, a.s, a.qsum); 1, 2, 4, 8: it quantises its token rows itself
// with the whole block (block_quant, rows padded to FQM, at most 8 tokens);
// 16: itself, one warp per row (up to 16 tokens).
constexpr int kFqWarpRows = 16;
constexpr int kFqVmax = 16;   // 16-byte vectors per thread and row in block_quant

template <int NT, int R, Epi EPI, typename T, bool SMEMW, int FQM>
__global__ void __launch_bounds__(kThreads) tgemm_mma_kernel(TGemmArgs a) {
  constexpr bool FQ = FQM != 0;
  __shared__ int red[R][16][NT * 8];
  __shared__ float s_sm[FQ ? NT * 8 : 1];
  __shared__ int qsum_sm[FQ ? NT * 8 : 1];
  extern __shared__ uint4 wsm[];     // SMEMW: [R][16][pitch4] weight slice; FQ: then [NT*8][fq_pitch] codes,
                                     // then the token rows [rows][K] in the activation dtype
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * 16;
  const int m0 = blockIdx.y * NT * 8;
  const int K = a.K, N = a.N, M = a.M;
  const int wpr = K / 16;            // packed words per row
  const int nkseg = ceil_div(K, 256);
  const int wpr4 = wpr / 4, pitch4 = wsm_pitch4(wpr);

  if constexpr (SMEMW) {             // weights do not depend on the predecessor
    for (int idx = threadIdx.x; idx < R * 16 * wpr4; idx += kThreads) {
      const int r = idx / (16 * wpr4), rem = idx - r * 16 * wpr4;
      const int row = rem / wpr4, c4 = rem - row * wpr4;
      const bool ok = n0 + row < N;
      const uint32_t* src = ok ? a.w[r] + (size_t)(n0 + row) * wpr + c4 * 4 : a.w[r];
      cp_async16(&wsm[(r * 16 + row) * pitch4 + c4], src, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i < R * 16 * NT * 8; i += kThreads) (&red[0][0][0])[i] = 0;
  int8_t* qs = reinterpret_cast<int8_t*>(wsm + (SMEMW ? R * 16 * pitch4 : 0));
  const int qpitch = fq_pitch(K);
  if constexpr (FQM >= 1 && FQM <= 8) {   // the whole block quantises the (at most 8) token rows
    __shared__ double red_d[kWarps];
    __shared__ uint32_t red_u[kWarps];
    __shared__ int red_i[kWarps];
    constexpr int kTpr = kThreads / FQM;
    const int m_row = threadIdx.x / kTpr, lt = threadIdx.x - m_row * kTpr;
    const int nvec = (int)(K * sizeof(T) / 16);
    const uint4* xg = reinterpret_cast<const uint4*>(static_cast<const T*>(a.x) + (size_t)m_row * K);
    uint4 raw[kFqVmax];
    uint32_t have = 0;
#pragma unroll
    for (int j = 0; j < kFqVmax; ++j) {
      const int v = lt + kTpr * j;
      raw[j] = make_uint4(0u, 0u, 0u, 0u);
      if (m_row < M && v < nvec) {
        have |= 1u << j;
        raw[j] = __ldcg(xg + v);   // coherent: the previous kernel may have written x while this one started
      }
    }
    const BlockRed red{red_d, red_u, red_i};
    block_quant<T, FQM, kThreads, kFqVmax>(raw, have, M, K, a.gain, a.eps, qs, qpitch, s_sm, red);
    if (threadIdx.x < M) qsum_sm[threadIdx.x] = block_qsum<FQM, kThreads>(red, threadIdx.x);
    __syncthreads();
    if (blockIdx.x == 0 && a.q_out != nullptr) {   // one CTA also hands the codes out
      for (int i = threadIdx.x; i < M * K / 16; i += kThreads) {
        const int m = i / (K / 16), c16 = i - m * (K / 16);
        *reinterpret_cast<uint4*>(a.q_out + (size_t)m * K + c16 * 16) =
            *reinterpret_cast<const uint4*>(qs + (size_t)m * qpitch + c16 * 16);
      }
      if (threadIdx.x < M) {
        if (a.s_out) a.s_out[threadIdx.x] = s_sm[threadIdx.x];
        if (a.qsum_out) a.qsum_out[threadIdx.x] = qsum_sm[threadIdx.x];
      }
    }
  } else if constexpr (FQM == kFqWarpRows) {   // quantise this CTA's token rows, one warp per row
    const int nvec = (int)(K * sizeof(T) / 16);
    const int rows = min(NT * 8, M - m0);
    uint4* xs = reinterpret_cast<uint4*>(qs + (size_t)NT * 8 * qpitch);
    const uint4* xg = reinterpret_cast<const uint4*>(static_cast<const T*>(a.x) + (size_t)m0 * K);
    for (int i = threadIdx.x; i < rows * nvec; i += kThreads) cp_async16(xs + i, xg + i, true);
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    for (int mc = warp; mc < rows; mc += kWarps) {
      const int m = m0 + mc;
      const uint4* xr = xs + (size_t)mc * nvec;
      int8_t* qr = qs + (size_t)mc * qpitch;
      const RowCode rc = a.gain != nullptr ? quant_row<T, true, false>(xr, nvec, K, a.gain, a.eps, qr, lane)
                                           : quant_row<T, false, false>(xr, nvec, K, nullptr, a.eps, qr, lane);
      if (lane == 0) {
        s_sm[mc] = rc.scale;
        qsum_sm[mc] = rc.qsum;
      }
      if (blockIdx.x == 0 && a.q_out != nullptr) {   // one CTA also hands the codes out
        __syncwarp();
        for (int i = lane; i < K / 16; i += 32)
          *reinterpret_cast<uint4*>(a.q_out + (size_t)m * K + i * 16) = *reinterpret_cast<const uint4*>(qr + i * 16);
        if (lane == 0) {
          if (a.s_out) a.s_out[m] = rc.scale;
          if (a.qsum_out) a.qsum_out[m] = rc.qsum;
        }
      }
    }
  }
  if constexpr (SMEMW) asm volatile("cp.async.wait_all;" ::: "memory");
  if constexpr (SMEMW || FQ) __syncthreads();

  int acc[R][NT][4];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][j][e] = 0;

  for (int seg = warp; seg < nkseg; seg += kWarps) {
    const int w0 = seg * 16 + 4 * t;   // first packed word of this lane
    uint4 wa[R], wb[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if constexpr (SMEMW) {
        const bool in = w0 < wpr;    // wpr % 4 == 0: a 16-byte group is all in or all out
        wa[r] = in ? wsm[(r * 16 + g) * pitch4 + (w0 >> 2)] : make_uint4(0u, 0u, 0u, 0u);
        wb[r] = in ? wsm[(r * 16 + g + 8) * pitch4 + (w0 >> 2)] : make_uint4(0u, 0u, 0u, 0u);
      } else {
        const uint32_t* W = a.w[r];
        wa[r] = load_words4(W + (size_t)(n0 + g) * wpr, w0, wpr, n0 + g < N);
        wb[r] = load_words4(W + (size_t)(n0 + g + 8) * wpr, w0, wpr, n0 + g + 8 < N);
      }
    }
    uint4 act[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int m = m0 + 8 * j + g;
      const int8_t* qrow = FQ ? nullptr : a.q + (size_t)m * K;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        // bytes [64t + 16u, +16) of this segment = packed word w0 + u's 16 columns
        const bool ok = (m < M) && (w0 + u < wpr);
        if constexpr (FQ)
          act[j][u] = ok ? *reinterpret_cast<const uint4*>(qs + (size_t)(8 * j + g) * qpitch + (w0 + u) * 16)
                         : make_uint4(0u, 0u, 0u, 0u);
        else
          act[j][u] = ok ? __ldg(reinterpret_cast<const uint4*>(qrow + (size_t)(w0 + u) * 16))
                         : make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int u = i >> 1, sub = (i & 1) * 2;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t wg = u4get(wa[r], u), wg8 = u4get(wb[r], u);
        const uint32_t a0 = (wg >> (2 * sub)) & kLow2;
        const uint32_t a2 = (wg >> (2 * sub + 2)) & kLow2;
        const uint32_t a1 = (wg8 >> (2 * sub)) & kLow2;
        const uint32_t a3 = (wg8 >> (2 * sub + 2)) & kLow2;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          const uint32_t b0 = u4get(act[j][u], sub), b1 = u4get(act[j][u], sub + 1);
          mma_u8s8(acc[r][j], a0, a1, a2, a3, b0, b1);
        }
      }
    }
  }
  __syncthreads();   // red[] zeroed
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      atomicAdd(&red[r][g][8 * j + 2 * t], acc[r][j][0]);
      atomicAdd(&red[r][g][8 * j + 2 * t + 1], acc[r][j][1]);
      atomicAdd(&red[r][g + 8][8 * j + 2 * t], acc[r][j][2]);
      atomicAdd(&red[r][g + 8][8 * j + 2 * t + 1], acc[r][j][3]);
    }
  __syncthreads();

  // ---------------------------------------------------------------- epilogue
  constexpr int kCols = NT * 8;
  auto row_scale = [&](int mc) { return FQ ? s_sm[mc] : a.s[m0 + mc]; };
  auto row_qsum = [&](int mc) { return FQ ? qsum_sm[mc] : a.qsum[m0 + mc]; };
  if constexpr (EPI == Epi::kStore || EPI == Epi::kAcc) {
    for (int idx = threadIdx.x; idx < R * 16 * kCols; idx += kThreads) {
      const int row = idx & 15, r = (idx >> 4) % R, mc = idx / (16 * R);
      const int n = n0 + row, m = m0 + mc;
      if (n >= N || m >= M) continue;
      const int accv = red[r][row][mc] - row_qsum(mc);
      if constexpr (EPI == Epi::kAcc) {
        static_cast<int32_t*>(a.out)[(size_t)m * a.ldo + r * N + n] = accv;
      } else {
        float v = rescale_acc(accv, *a.gamma[r], row_scale(mc));
        if (a.bias[r] != nullptr) v += a.bias[r][n];
        if (a.residual != nullptr) v += to_f32(static_cast<const T*>(a.residual)[(size_t)m * N + n]);
        static_cast<T*>(a.out)[(size_t)m * a.ldo + r * N + n] = from_f32<T>(v);
      }
    }
  } else if constexpr (EPI == Epi::kScanStep) {
    for (int idx = threadIdx.x; idx < 16 * kCols; idx += kThreads) {
      const int row = idx & 15, mc = idx >> 4;
      const int n = n0 + row, m = m0 + mc;
      if (n >= N || m >= M) continue;
      float pre[3];
#pragma unroll
      for (int r = 0; r < 3; ++r) {
        float v = rescale_acc(red[r][row][mc] - row_qsum(mc), *a.gamma[r], row_scale(mc));
        if (a.bias[r] != nullptr) v += a.bias[r][n];
        pre[r] = round_to<T>(v);   // the pre-activations are a storage point
        if (a.pre_out != nullptr) static_cast<T*>(a.pre_out)[((size_t)m * 3 + r) * N + n] = from_f32<T>(pre[r]);
      }
      float* hp = a.h + (size_t)m * N + n;
      float hn = *hp;
      const float og = mlgru_step(pre[0], pre[1], pre[2], hn);
      *hp = hn;
      static_cast<T*>(a.out)[(size_t)m * a.ldo + n] = from_f32<T>(og);
    }
  } else {  // kGlu
    for (int idx = threadIdx.x; idx < 16 * kCols; idx += kThreads) {
      const int row = idx & 15, mc = idx >> 4;
      const int n = n0 + row, m = m0 + mc;
      if (n >= N || m >= M) continue;
      float uv[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float v = rescale_acc(red[r][row][mc] - row_qsum(mc), *a.gamma[r], row_scale(mc));
        if (a.bias[r] != nullptr) v += a.bias[r][n];
        uv[r] = v;
      }
      static_cast<T*>(a.out)[(size_t)m * a.ldo + n] = from_f32<T>(siluf_(uv[0]) * uv[1]);
    }
  }
}

constexpr size_t kFqBytes = 128 * 1024;   // fused-quantisation limit: codes + staged token rows

template <int NT, int R, Epi EPI, typename T, bool SMEMW, int FQM>
cudaError_t launch_variant(const TGemmArgs& a, dim3 grid, size_t smem, cudaStream_t stream) {
  auto kern = tgemm_mma_kernel<NT, R, EPI, T, SMEMW, FQM>;
  if (smem > 0) {   // the default limit covers static + dynamic together, so opt in whenever there is any
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(kern, grid, dim3(kThreads), smem, stream, a);
}

template <int NT, int R, Epi EPI, typename T>
cudaError_t launch_one(const TGemmArgs& a, cudaStream_t stream) {
  dim3 grid(ceil_div(a.N, 16), ceil_div(a.M, NT * 8));
  const int wpr = a.K / 16;
  const size_t wbytes = (size_t)R * 16 * wsm_pitch4(wpr) * 16;
  const bool fq = a.x != nullptr;
  // (Sizing the codes buffer for the M rows alone measured slower on one B200
  // for chains of single-token calls: 3.9 -> 4.9 us per 2048 x 2048 call.)
  const size_t qbytes = fq ? (size_t)NT * 8 * fq_pitch(a.K) + (size_t)std::min(a.M, NT * 8) * a.K * sizeof(T) : 0;
  if (fq && (NT > 2 || qbytes > kFqBytes)) return cudaErrorInvalidValue;
  // the weight slice goes to shared memory when it fits next to the codes
  const bool smemw = wpr % 4 == 0 && wbytes <= 100 * 1024 && wbytes + qbytes <= 200 * 1024;
  const size_t smem = (smemw ? wbytes : 0) + qbytes;
  if (!fq) return smemw ? launch_variant<NT, R, EPI, T, true, 0>(a, grid, smem, stream)
                        : launch_variant<NT, R, EPI, T, false, 0>(a, grid, smem, stream);
  if constexpr (NT == 1) {   // the whole block on each row when every thread's share fits its registers
    const int mpad = a.M <= 1 ? 1 : (a.M <= 2 ? 2 : (a.M <= 4 ? 4 : 8));
    const int nvec = (int)(a.K * sizeof(T) / 16);
    if (ceil_div(nvec, kThreads / mpad) <= kFqVmax) {
      switch (mpad) {
        case 1: return smemw ? launch_variant<NT, R, EPI, T, true, 1>(a, grid, smem, stream)
                             : launch_variant<NT, R, EPI, T, false, 1>(a, grid, smem, stream);
        case 2: return smemw ? launch_variant<NT, R, EPI, T, true, 2>(a, grid, smem, stream)
                             : launch_variant<NT, R, EPI, T, false, 2>(a, grid, smem, stream);
        case 4: return smemw ? launch_variant<NT, R, EPI, T, true, 4>(a, grid, smem, stream)
                             : launch_variant<NT, R, EPI, T, false, 4>(a, grid, smem, stream);
        default: return smemw ? launch_variant<NT, R, EPI, T, true, 8>(a, grid, smem, stream)
                              : launch_variant<NT, R, EPI, T, false, 8>(a, grid, smem, stream);
      }
    }
  }
  return smemw ? launch_variant<NT, R, EPI, T, true, kFqWarpRows>(a, grid, smem, stream)
               : launch_variant<NT, R, EPI, T, false, kFqWarpRows>(a, grid, smem, stream);
}

template <int NT, typename T>
cudaError_t launch_nt(const TGemmArgs& a, Epi epi, cudaStream_t stream) {
  switch (epi) {
    case Epi::kStore:
      if (a.nseg == 1) return launch_one<NT, 1, Epi::kStore, T>(a, stream);
      if (a.nseg == 2) return launch_one<NT, 2, Epi::kStore, T>(a, stream);
      return launch_one<NT, 3, Epi::kStore, T>(a, stream);
    case Epi::kAcc: return launch_one<NT, 1, Epi::kAcc, T>(a, stream);
    case Epi::kScanStep: return launch_one<NT, 3, Epi::kScanStep, T>(a, stream);
    case Epi::kGlu: return launch_one<NT, 2, Epi::kGlu, T>(a, stream);
  }
  return cudaErrorInvalidValue;
}

// At most 32 tokens per CTA: above that a second grid row takes the next 32
// tokens and reads the same weight slice again (from L2). A 64-token CTA would
// keep eight token tiles of fragments and its accumulators in registers and
// spill (the f|c|g step needs 255 registers).
template <typename T>
cudaError_t launch_t(const TGemmArgs& a, Epi epi, cudaStream_t stream) {
  if (a.M <= 8) return launch_nt<1, T>(a, epi, stream);
  if (a.M <= 16) return launch_nt<2, T>(a, epi, stream);
  return launch_nt<4, T>(a, epi, stream);
}

}  // namespace

bool tgemm_mma_fused_quant_supported(int M, int K, int esize) {
  const int nt = M <= 8 ? 1 : 2;
  return M >= 1 && M <= 16 && (size_t)nt * 8 * fq_pitch(K) + (size_t)M * K * esize <= kFqBytes;
}

cudaError_t launch_tgemm_mma(const TGemmArgs& a, Epi epi, mmf_dtype dt, cudaStream_t stream) {
  if (a.M == 0 || a.N == 0) return cudaSuccess;
  return dt == MMF_BF16 ? launch_t<bf16>(a, epi, stream) : launch_t<float>(a, epi, stream);
}

}  // namespace mmf
