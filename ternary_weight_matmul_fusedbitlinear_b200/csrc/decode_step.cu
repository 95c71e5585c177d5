// One decode step (T = 1) of a stack of MatMul-free blocks in one kernel
// launch (sm_100a).
//
// "MatMul-free language models" (DataCamp blog), sections "Replacing MatMul
// with ternary operations" and "Core components: MLGRU and GLU"; the hysenlabs
// review, sections "FusedBitLinear" and "HGRN attention". A layer is four
// FusedBitLinear stages, each of which normalises and quantises its whole
// input rows before it accumulates against ternary weights:
//   S0  x  -> f|c|g (3 x d rows) -> MLGRU step: h = f h + (1 - f) c, o' = g h
//   S1  o' -> o (d rows) + x                            -> y1
//   S2  y1 -> gate|up (2 x I rows) -> SiLU(gate) * up   -> p
//   S3  p  -> down (d rows) + y1                        -> x of the next layer (y after the last)
//
// Why one launch: a decode step is a chain of 4 L dependent stages. Each
// stage needs every element of the previous stage's output (the RMS and the
// absmax scale are reductions over the whole row), while the weights it
// streams (a few MB) take HBM about a microsecond. The step's time is the
// chain's latency, so the launch is built around it:
//   * Stage outputs travel through buffers owned by the recurrent state. Their
//     elements are reset to all-ones bits (a NaN pattern that no stage ever
//     stores) one launch ahead, and a consumer re-reads its input rows until no
//     element holds that pattern: the data are their own ready flags (each
//     element is written once, by one aligned store). There is no grid
//     barrier, no fence and no flag round trip. Two sets of buffers alternate
//     by a per-layer launch parity kept in the state: a launch writes set P
//     and resets set 1 - P for the next launch.
//   * A CTA owns the 16-row tiles b, b + G, ... of every stage's matrices. Its
//     weight slices stream into a shared-memory ring by 1-D bulk copies
//     (cp.async.bulk, one per tile and segment) several stages ahead. Weights
//     do not depend on activations, so the HBM stream runs ahead of the chain.
//     (L2 prefetches further ahead measured slower: their instructions share
//     the SM's memory pipeline with the chain's own loads and stores.)
//   * Every CTA quantises the whole input rows itself with all 16 warps: the
//     rows go to registers, the fp64 sum of squares and the max are reduced
//     over the block in a fixed order (every CTA gets the same scale), and the
//     codes go to shared memory with the same fp32 steps as the standalone
//     quantiser. The contraction is mma.sync m16n8k32 (stored codes w + 1 as
//     u8 against s8 activations; the row's code sum is subtracted after),
//     its units spread evenly over the warps by a per-stage plan worked out
//     once at kernel start.
// Launch: cooperative, one CTA of 512 threads per SM, so every CTA is resident
// and every wait ends. Each wait is also bounded: on timeout a CTA records
// status code 5 (input rows) or 6 (weight slice), raises the state's abort word
// so that the other CTAs leave as well, lets its copies land and returns. The
// state must then be reset before its next decode step.
#include "kernels.cuh"
#include "quant_row.cuh"
#include "tma.cuh"

namespace mmf {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kVmax = 16;            // 16-byte input vectors per thread and stage
constexpr uint32_t kLow2 = 0x03030303u;

struct StageGeom {
  int nseg, N, K, mat0, gain;
};
__host__ __device__ __forceinline__ StageGeom stage_geom(int s, int d, int I) {
  if (s == 0) return StageGeom{3, d, d, 0, 0};
  if (s == 1) return StageGeom{1, d, d, 3, 1};
  if (s == 2) return StageGeom{2, I, d, 4, 2};
  return StageGeom{1, d, I, 6, 3};
}
// 16-row tiles of an N-row matrix that CTA b of G owns (tiles b, b + G, ...).
__host__ __device__ __forceinline__ int tiles_of(int N, int b, int G) {
  const int nt = N / 16;
  return b < nt ? (nt - b + G - 1) / G : 0;
}

// Byte offset of region r (0: o', 1: y1, 2: p, 3: next layer's x) inside one
// buffer set; 4 bytes per element whatever the dtype, so regions never move.
__host__ __device__ __forceinline__ size_t region_off(int r, int M, int d, int I) {
  const size_t md = (size_t)M * d * 4;
  return r == 0 ? 0 : (r == 1 ? md : (r == 2 ? 2 * md : 2 * md + (size_t)M * I * 4));
}

// Regions are laid out for the inner size the buffers were allocated for (xI >= I).
__device__ __forceinline__ uint8_t* xregion(const DecodeStepArgs& a, int l, int set, int r) {
  return a.xbuf + (size_t)(a.layer0 + l) * a.xlayer_bytes + (size_t)set * a.xset_bytes + region_off(r, a.M, a.d, a.xI);
}

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

__device__ __forceinline__ uint4 ld_relaxed_v4(const void* p) {
  uint4 r;
  asm volatile("ld.relaxed.gpu.global.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p)
               : "memory");
  return r;
}
__device__ __forceinline__ int ld_relaxed_i32(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One element of a stage output: published with a relaxed store (read by
// other CTAs' relaxed loads), and the same position of the other buffer set
// reset to all-ones bits for the next launch.
__device__ __forceinline__ void publish(bf16* cur, bf16* next, float v) {
  const bf16 h = from_f32<bf16>(v);
  const unsigned short u = *reinterpret_cast<const unsigned short*>(&h);
  asm volatile("st.relaxed.gpu.global.b16 [%0], %1;" ::"l"(cur), "h"(u) : "memory");
  *reinterpret_cast<unsigned short*>(next) = 0xffffu;
}
__device__ __forceinline__ void publish(float* cur, float* next, float v) {
  asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(cur), "r"(__float_as_uint(v)) : "memory");
  *reinterpret_cast<uint32_t*>(next) = 0xffffffffu;
}

// Whether a 16-byte vector of stage output still holds an unwritten element.
template <typename T> __device__ __forceinline__ bool has_unset(const uint4& v);
template <> __device__ __forceinline__ bool has_unset<bf16>(const uint4& v) {
  return (__vcmpeq2(v.x, 0xffffffffu) | __vcmpeq2(v.y, 0xffffffffu) | __vcmpeq2(v.z, 0xffffffffu) |
          __vcmpeq2(v.w, 0xffffffffu)) != 0u;
}
template <> __device__ __forceinline__ bool has_unset<float>(const uint4& v) {
  return v.x == ~0u || v.y == ~0u || v.z == ~0u || v.w == ~0u;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// This CTA's share of one stage type (S0..S3 repeat in every layer), worked
// out once at kernel start so that no integer division sits on the chain.
struct StagePlan {
  int ntl;                 // 16-row tiles of each segment (tiles b, b + G, ...)
  int nk;                  // 128-column units per row
  short a0[kWarps];        // warp w's units: segment a0, column block c0, n units (segment-major)
  short c0[kWarps];
  short n[kWarps];
};

struct Smem {
  StagePlan plan[4];
  int red[kDecodeTiles][3][16][8];      // per tile, segment, row, token: exact int32 partial sums
  double red_d[kWarps];
  uint32_t red_u[kWarps];
  int red_i[kWarps];
  float scale[8];
  float res_x[kDecodeTiles * 16 * 8];   // block input x of this CTA's d-channels (S1 residual)
  float res_y1[kDecodeTiles * 16 * 8];  // y1 of this CTA's d-channels (S3 residual)
  float gam[kDecodeMaxLayers][7];
  unsigned par[kDecodeMaxLayers];
  uint64_t slot_bar[kDecodeMaxSlots];
  int fail_code;                        // 5: an input row never arrived, 6: a weight slot never landed
};

// One warp: start the bulk copies of stage q's weight slice into its ring slot.
// A 16-row tile of one matrix is contiguous in memory (rows of K/4 bytes), so
// each (tile, segment) is one copy, landing as 16 dense rows. (A copy per row,
// to pad the rows in shared memory, floods the SM's memory pipeline with copy
// instructions and stalls the stores and loads of the chain behind them.)
__device__ void fill_slot(const DecodeStepArgs& a, const DecodeLayerDesc* desc, uint8_t* slots, Smem& sm, int q,
                          int lane) {
  const int l = q >> 2, s = q & 3;
  const StageGeom g = stage_geom(s, a.d, a.I);
  const int ntl = sm.plan[s].ntl;
  const int tile_bytes = 16 * (g.K / 4);
  const int slot = q % a.nslot;
  uint8_t* dst0 = slots + (size_t)slot * a.slot_bytes;
  const int ncopy = ntl * g.nseg;
  if (lane == 0) {
    if (ncopy > 0) mbar_arrive_expect_tx(&sm.slot_bar[slot], (uint32_t)(ncopy * tile_bytes));
    else mbar_arrive(&sm.slot_bar[slot]);
  }
  __syncwarp();
  for (int i = lane; i < ncopy; i += 32) {   // i = tile * nseg + segment
    const int ti = i / g.nseg, r = i - ti * g.nseg;
    const int t = blockIdx.x + ti * gridDim.x;
    const uint8_t* src = reinterpret_cast<const uint8_t*>(desc[l].w[g.mat0 + r]) + (size_t)t * tile_bytes;
    bulk_g2s(dst0 + (size_t)i * tile_bytes, src, (uint32_t)tile_bytes, &sm.slot_bar[slot]);
  }
}

// Accumulate this CTA's tiles of one stage into red[ti][r][row][token].
//
// The stored code c = w + 1 of column 16 j + 4 p + b sits at bits 8 b + 2 p of
// packed word j, so word & (0x03030303 << 2 p) holds c 4^p in byte b: one
// logic operation per 4 codes and no shift. Each field position p
// accumulates into its own sums, which are multiples of 4^p and are scaled
// back exactly by an arithmetic shift: acc = sum_p (chain_p >> 2 p).
// m16n8k32 MMAs take rows g and g + 8 of a tile segment against tokens 2 t,
// 2 t + 1. A unit is 128 columns of a segment (the lane's two packed words of
// each of the two rows) and four MMAs, one per field position; consecutive
// units go to two sets of chains so that two MMAs of a chain are never back to
// back. Warp w takes the contiguous units [w U / 16, (w + 1) U / 16) of the
// segment-major order (the stage plan), so every warp gets an equal share
// whatever the CTA's tile count.
__device__ __forceinline__ void mma_unit(int (&acc)[4][4], const uint8_t* wrow, int rowb, const int8_t* qrow, int c,
                                         int K, int t, bool tok) {
  const bool kin = c * 128 + t * 32 < K;   // K % 64 == 0: a last unit of 64 columns uses lanes t < 2
  uint2 wa = make_uint2(0u, 0u), wb = wa;
  uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
  if (kin) {
    wa = *reinterpret_cast<const uint2*>(wrow + c * 32);
    wb = *reinterpret_cast<const uint2*>(wrow + (size_t)8 * rowb + c * 32);
    if (tok) {   // token g's codes of the lane's two words
      x0 = *reinterpret_cast<const uint4*>(qrow + c * 128);
      x1 = *reinterpret_cast<const uint4*>(qrow + c * 128 + 16);
    }
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t m = kLow2 << (2 * p);
    mma_u8s8(acc[p], wa.x & m, wb.x & m, wa.y & m, wb.y & m, u4get(x0, p), u4get(x1, p));
  }
}

// Tile of segment index a of a stage with nseg segments per tile (a < 9, nseg <= 3), without a division.
__device__ __forceinline__ int seg_tile(int a, int nseg) { return nseg == 1 ? a : (nseg == 2 ? a >> 1 : (a * 11) >> 5); }

__device__ __forceinline__ void stage_mma(const uint8_t* slot, const int8_t* qs, int qpitch, int M, int K,
                                          const StagePlan& pl, int nseg, int (*red)[3][16][8]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rowb = K / 4, nk = pl.nk;
  const bool tok = g < M;
  const int8_t* qrow = qs + (size_t)(tok ? g : 0) * qpitch + t * 32;
  int left = pl.n[warp], c0 = pl.c0[warp];
  for (int a = pl.a0[warp]; left > 0; ++a, c0 = 0) {   // the tile segments this warp's units touch
    const int c1 = min(nk, c0 + left);
    left -= c1 - c0;
    const uint8_t* wrow = slot + ((size_t)a * 16 + g) * rowb + t * 8;
    int acc0[4][4], acc1[4][4];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc0[p][e] = acc1[p][e] = 0;
    int c = c0;
    for (; c + 1 < c1; c += 2) {
      mma_unit(acc0, wrow, rowb, qrow, c, K, t, tok);
      mma_unit(acc1, wrow, rowb, qrow, c + 1, K, t, tok);
    }
    if (c < c1) mma_unit(acc0, wrow, rowb, qrow, c, K, t, tok);
    const int ti = seg_tile(a, nseg), r = a - ti * nseg;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = 2 * t + (e & 1);
      if (col < M) {
        int v = 0;
#pragma unroll
        for (int p = 0; p < 4; ++p) v += (acc0[p][e] + acc1[p][e]) >> (2 * p);
        atomicAdd(&red[ti][r][g + 8 * (e >> 1)][col], v);
      }
    }
  }
}

// Give up: record `code`, raise the abort word, let this CTA's weight copies
// in flight land (bounded), and return.
__device__ void give_up(const DecodeStepArgs& a, Smem& sm, int code, int q_first, int q_end) {
  if (threadIdx.x == 0) {
    if (a.status) atomicExch(a.status, code);
    atomicExch(a.abort_word, 1);
    for (int q = q_first; q < q_end; ++q) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&sm.slot_bar[q % a.nslot], (uint32_t)(q / a.nslot) & 1u) &&
             clock64() - t0 < a.wait_cycles) {
      }
    }
  }
  __syncthreads();
}

template <typename T, int MPAD>
__global__ void __launch_bounds__(kThreads, 1) decode_step_kernel(const __grid_constant__ DecodeStepArgs a) {
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ Smem sm;
  using V = Vec<T>;
  constexpr int E = V::E;
  constexpr int kTpr = kThreads / MPAD;     // threads per token row in the quantisation
  const BlockRed red{sm.red_d, sm.red_u, sm.red_i};
  DecodeLayerDesc* desc = reinterpret_cast<DecodeLayerDesc*>(dsm);
  int8_t* codes = reinterpret_cast<int8_t*>(dsm + a.desc_bytes);
  uint8_t* slots = dsm + a.desc_bytes + a.codes_bytes;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x, G = gridDim.x;
  const int M = a.M, d = a.d, I = a.I, L = a.L;
  const int nq = 4 * L;
  const int qpitch = a.qpitch;

  if (tid == 0) {
    sm.fail_code = 0;
    for (int s = 0; s < a.nslot; ++s) mbar_init(&sm.slot_bar[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  {   // layer descriptors into shared memory (written before this launch)
    constexpr int kWords = sizeof(DecodeLayerDesc) / 8;
    for (int i = tid; i < L * kWords; i += kThreads)
      reinterpret_cast<uint64_t*>(desc)[i] = reinterpret_cast<const uint64_t*>(a.layer[i / kWords])[i % kWords];
  }
  if (tid < 4 * kWarps) {   // the stage plans: thread 16 s + w works out warp w's units of stage type s
    const int ps = tid / kWarps, pw = tid % kWarps;
    const StageGeom pg = stage_geom(ps, d, I);
    const int ntl = tiles_of(pg.N, b, G), nk = ceil_div(pg.K, 128);
    const int total = ntl * pg.nseg * nk;
    const int u0 = pw * total / kWarps, u1 = (pw + 1) * total / kWarps;
    sm.plan[ps].a0[pw] = (short)(u0 / nk);
    sm.plan[ps].c0[pw] = (short)(u0 % nk);
    sm.plan[ps].n[pw] = (short)(u1 - u0);
    if (pw == 0) {
      sm.plan[ps].ntl = ntl;
      sm.plan[ps].nk = nk;
    }
  }
  __syncthreads();
  for (int i = tid; i < L * 7; i += kThreads) sm.gam[i / 7][i % 7] = *desc[i / 7].gamma[i % 7];
  // the weight stream does not depend on the previous kernel: start it first
  int q_issued = 0;   // stages whose ring fill has been issued
  if (warp == kWarps - 1) {
    for (int q = 0; q < a.nslot && q < nq; ++q) fill_slot(a, desc, slots, sm, q, lane);
  }
  q_issued = a.nslot < nq ? a.nslot : nq;
  pdl_wait();
  if (tid < L) sm.par[tid] = a.parity[a.layer0 + tid] & 1u;
  __syncthreads();

  const int m_row = tid / kTpr, lt = tid - m_row * kTpr;   // quantisation: this thread's token row
  const bool row_ok = m_row < M;
  // epilogue: thread tid owns output row e_row of tile e_ti for token e_m (tid < ntl 16 M)
  const int e_ti = tid / (16 * M), e_rem = tid - e_ti * 16 * M;
  const int e_m = e_rem >> 4, e_row = e_rem & 15;
  const int e_n = (b + e_ti * G) * 16 + e_row;

  for (int q = 0; q < nq; ++q) {
    const int l = q >> 2, s = q & 3;
    const StageGeom g = stage_geom(s, d, I);
    const DecodeLayerDesc& D = desc[l];
    const int ntl = sm.plan[s].ntl;
    const int par = (int)sm.par[l];
    const int K = g.K, N = g.N;
    int(*red_q)[3][16][8] = sm.red;
    for (int i = tid; i < kDecodeTiles * 3 * 16 * 8; i += kThreads) (&red_q[0][0][0][0])[i] = 0;

    // ---------------------------------------------------- epilogue operands that need no input row
    const int nout = ntl * 16 * M;
    const bool has_out = tid < nout;
    float* hp = a.h + ((size_t)(a.layer0 + l) * M + e_m) * d + e_n;
    float hval = 0.0f, bias[3] = {0.0f, 0.0f, 0.0f};
    if (has_out) {
      if (s == 0) hval = *hp;
      for (int r = 0; r < g.nseg; ++r)
        if (D.bias[g.mat0 + r] != nullptr) bias[r] = D.bias[g.mat0 + r][e_n];
    }

    // ---------------------------------------------------- input rows -> registers
    const uint8_t* in;
    bool poll = true;
    if (s == 0) {
      if (l == 0) {
        in = static_cast<const uint8_t*>(a.x);
        poll = false;
      } else {
        in = xregion(a, l - 1, (int)sm.par[l - 1], 3);
      }
    } else {
      in = xregion(a, l, par, s - 1);
    }
    const int nvec = K * (int)sizeof(T) / 16;
    const uint8_t* src = in + (size_t)(row_ok ? m_row : 0) * K * sizeof(T);
    uint4 raw[kVmax];
    uint32_t pend = 0;
#pragma unroll
    for (int j = 0; j < kVmax; ++j) {
      raw[j] = make_uint4(0u, 0u, 0u, 0u);
      if (row_ok && lt + kTpr * j < nvec) pend |= 1u << j;
    }
    const uint32_t have = pend;
    bool failed = false;
    if (!poll) {
#pragma unroll
      for (int j = 0; j < kVmax; ++j)
        if (have & (1u << j)) raw[j] = __ldcg(reinterpret_cast<const uint4*>(src) + lt + kTpr * j);
    } else {
      long long t0 = 0;
      while (pend != 0u) {
#pragma unroll
        for (int j = 0; j < kVmax; ++j)
          if (pend & (1u << j)) {
            raw[j] = ld_relaxed_v4(src + (size_t)(lt + kTpr * j) * 16);
            if (!has_unset<T>(raw[j])) pend &= ~(1u << j);
          }
        if (pend == 0u) break;
        const long long now = clock64();
        if (t0 == 0) t0 = now;
        else if (now - t0 > a.wait_cycles || ld_relaxed_i32(a.abort_word) != 0) {
          failed = true;
          break;
        }
      }
    }
    // this stage's weight slice (issued stages ahead, normally landed long ago)
    const int slot = q % a.nslot;
    bool got = mbar_try_wait(&sm.slot_bar[slot], (uint32_t)(q / a.nslot) & 1u);
    if (!got && !failed) {
      const long long t0 = clock64();
      while (!(got = mbar_try_wait(&sm.slot_bar[slot], (uint32_t)(q / a.nslot) & 1u))) {
        if (clock64() - t0 > a.wait_cycles) break;
      }
    }
    if (failed || !got) atomicMax(&sm.fail_code, failed ? 5 : 6);

    // ---------------------------------------------------- RMSNorm + absmax int8 codes, whole block
    // (its first barrier is also the vote on giving up)
    const float* gain = D.gain[g.gain];
    if (!block_quant<T, MPAD, kThreads, kVmax>(raw, have, M, K, gain, a.eps, codes, qpitch, sm.scale, red,
                                               failed || !got)) {
      give_up(a, sm, sm.fail_code, q, q_issued);
      return;
    }
    if (s == 0 || s == 2) {   // keep this CTA's channels of x (S1 residual) / y1 (S3 residual)
      float* res = s == 0 ? sm.res_x : sm.res_y1;
#pragma unroll
      for (int j = 0; j < kVmax; ++j) {
        if (!(have & (1u << j))) break;
        const int v = lt + kTpr * j;
        const int t16 = (v * E) >> 4;   // this CTA's tiles are b, b + G, b + 2 G (d <= 48 G)
        const int ti = t16 == b ? 0 : (t16 == b + G ? 1 : (t16 == b + 2 * G ? 2 : -1));
        if (ti >= 0) {
#pragma unroll
          for (int i = 0; i < E; ++i) res[(ti * 16 + ((v * E + i) & 15)) * 8 + m_row] = V::val(raw[j], i);
        }
      }
    }   // read by the epilogue of a later stage, after several barriers
    if (a.dbg.q[s] != nullptr && b == 0) {   // debug: this stage's codes and scales (one launch, one layer)
      for (int i = tid; i < M * K / 16; i += kThreads) {
        const int m = i / (K / 16), c16 = i - m * (K / 16);
        *reinterpret_cast<uint4*>(a.dbg.q[s] + (size_t)m * K + c16 * 16) =
            *reinterpret_cast<const uint4*>(codes + (size_t)m * qpitch + c16 * 16);
      }
      if (tid < M && a.dbg.scale[s] != nullptr) a.dbg.scale[s][tid] = sm.scale[tid];
    }

    // ---------------------------------------------------- the contraction
    stage_mma(slots + (size_t)slot * a.slot_bytes, codes, qpitch, M, K, sm.plan[s], g.nseg, red_q);
    __syncthreads();
    if (warp == kWarps - 1) {   // the slot is free: refill it `nslot` stages ahead (this warp has
      fence_proxy_async_smem();  // no epilogue work: at most 384 outputs per CTA)
      if (q + a.nslot < nq) fill_slot(a, desc, slots, sm, q + a.nslot, lane);
    }
    if (q + a.nslot < nq) q_issued = q + a.nslot + 1;

    // ---------------------------------------------------- epilogue: one output element per thread
    if (has_out) {
      const float sc = sm.scale[e_m];
      const int qs = block_qsum<MPAD, kThreads>(red, e_m);
      const size_t o_idx = (size_t)e_m * N + e_n;
      const bool skip = b == a.skip_cta && q == 0;   // test hook: one CTA never publishes its first stage
      if (s == 0) {
        float pre[3];
#pragma unroll
        for (int r = 0; r < 3; ++r) {
          pre[r] = round_to<T>(rescale_acc(red_q[e_ti][r][e_row][e_m] - qs, sm.gam[l][r], sc) + bias[r]);
          if (a.dbg.pre != nullptr) static_cast<T*>(a.dbg.pre)[((size_t)e_m * 3 + r) * d + e_n] = from_f32<T>(pre[r]);
        }
        const float og = mlgru_step(pre[0], pre[1], pre[2], hval);
        *hp = hval;
        if (!skip)
          publish(reinterpret_cast<T*>(xregion(a, l, par, 0)) + o_idx, reinterpret_cast<T*>(xregion(a, l, par ^ 1, 0)) + o_idx,
                  og);
        if (a.dbg.og != nullptr) static_cast<T*>(a.dbg.og)[o_idx] = from_f32<T>(og);
      } else if (s == 2) {
        float uv[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) uv[r] = rescale_acc(red_q[e_ti][r][e_row][e_m] - qs, sm.gam[l][4 + r], sc) + bias[r];
        const float p = siluf_(uv[0]) * uv[1];
        publish(reinterpret_cast<T*>(xregion(a, l, par, 2)) + o_idx, reinterpret_cast<T*>(xregion(a, l, par ^ 1, 2)) + o_idx, p);
        if (a.dbg.p != nullptr) static_cast<T*>(a.dbg.p)[o_idx] = from_f32<T>(p);
      } else {
        const float* res = s == 1 ? sm.res_x : sm.res_y1;
        const float v = rescale_acc(red_q[e_ti][0][e_row][e_m] - qs, sm.gam[l][g.mat0], sc) + bias[0] +
                        res[(e_ti * 16 + e_row) * 8 + e_m];
        if (s == 1) {
          publish(reinterpret_cast<T*>(xregion(a, l, par, 1)) + o_idx,
                  reinterpret_cast<T*>(xregion(a, l, par ^ 1, 1)) + o_idx, v);
          if (a.dbg.y1 != nullptr) static_cast<T*>(a.dbg.y1)[o_idx] = from_f32<T>(v);
        } else if (l == L - 1) {
          static_cast<T*>(a.y)[o_idx] = from_f32<T>(v);
        } else {
          publish(reinterpret_cast<T*>(xregion(a, l, par, 3)) + o_idx,
                  reinterpret_cast<T*>(xregion(a, l, par ^ 1, 3)) + o_idx, v);
        }
      }
    }
    // red, codes and the residual slices are reused by the next stage; the
    // barrier also keeps early warps from polling the next stage's input while
    // others still publish (without it: 0.75 vs 0.67 ms per 2.7B token)
    __syncthreads();
  }
  if (b == 0 && tid < L) a.parity[a.layer0 + tid] = sm.par[tid] ^ 1u;
}

struct Geom {
  int nslot, slot_bytes, qpitch;
  size_t desc_bytes, codes_bytes, smem;
};

constexpr size_t kDecodeSmemBudget = 214 * 1024;   // dynamic part; the static part is ~9 KB of the 227 KB

bool geometry(int M, int d, int I, int L, int esize, int G, Geom& g) {
  const int kmax = std::max(d, I);
  g.qpitch = kmax + 16;
  g.desc_bytes = (sizeof(DecodeLayerDesc) * (size_t)L + 127) / 128 * 128;
  g.codes_bytes = ((size_t)M * g.qpitch + 127) / 128 * 128;
  size_t slot = 0;
  for (int s = 0; s < 4; ++s) {
    const StageGeom sg = stage_geom(s, d, I);
    slot = std::max(slot, (size_t)tiles_of(sg.N, 0, G) * sg.nseg * 16 * (sg.K / 4));
  }
  g.slot_bytes = (int)((slot + 127) / 128 * 128);
  const size_t fixed = g.desc_bytes + g.codes_bytes;
  if (fixed + g.slot_bytes > kDecodeSmemBudget) return false;
  g.nslot = (int)std::min<size_t>(kDecodeMaxSlots, (kDecodeSmemBudget - fixed) / g.slot_bytes);
  g.smem = fixed + (size_t)g.nslot * g.slot_bytes;
  (void)esize;
  return true;
}

int mpad_of(int M) { return M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8)); }

template <typename T, int MPAD>
cudaError_t launch_typed(DecodeStepArgs a, const Geom& g, cudaStream_t stream) {
  auto kern = decode_step_kernel<T, MPAD>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, g.smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(decode_step_grid(a.d, a.I));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = g.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <typename T>
cudaError_t launch_t(const DecodeStepArgs& a, const Geom& g, cudaStream_t stream) {
  switch (mpad_of(a.M)) {
    case 1: return launch_typed<T, 1>(a, g, stream);
    case 2: return launch_typed<T, 2>(a, g, stream);
    case 4: return launch_typed<T, 4>(a, g, stream);
    default: return launch_typed<T, 8>(a, g, stream);
  }
}

}  // namespace

int decode_step_grid(int d, int I) { return std::min(num_sms(), std::max(d, I) / 16); }

size_t decode_xlayer_bytes(int M, int d, int I) {
  return (2 * (region_off(3, M, d, I) + (size_t)M * d * 4) + 255) / 256 * 256;
}

bool decode_step_supported(int M, int d, int I, int L, mmf_dtype dt) {
  if (M < 1 || M > 8 || L < 1 || L > kDecodeMaxLayers) return false;
  if (d < 64 || I < 64 || d % 64 != 0 || I % 64 != 0) return false;
  const int G = decode_step_grid(d, I);
  if (G < 1) return false;
  const int esize = dt == MMF_BF16 ? 2 : 4;
  const int mpad = mpad_of(M);
  const int tpr = kThreads / mpad;
  for (int s = 0; s < 4; ++s) {
    const StageGeom sg = stage_geom(s, d, I);
    if (tiles_of(sg.N, 0, G) > kDecodeTiles) return false;
    if (ceil_div(sg.K * esize / 16, tpr) > kVmax) return false;   // input vectors per thread
  }
  Geom g;
  return geometry(M, d, I, L, esize, G, g);
}

cudaError_t launch_decode_step(DecodeStepArgs a, mmf_dtype dt, cudaStream_t stream) {
  if (!decode_step_supported(a.M, a.d, a.I, a.L, dt)) return cudaErrorNotSupported;
  Geom g;
  geometry(a.M, a.d, a.I, a.L, dt == MMF_BF16 ? 2 : 4, decode_step_grid(a.d, a.I), g);
  a.nslot = g.nslot;
  a.slot_bytes = g.slot_bytes;
  a.qpitch = g.qpitch;
  a.desc_bytes = (int)g.desc_bytes;
  a.codes_bytes = (int)g.codes_bytes;
  if (a.xI < a.I) return cudaErrorInvalidValue;
  a.xlayer_bytes = decode_xlayer_bytes(a.M, a.d, a.xI);
  a.xset_bytes = a.xlayer_bytes / 2;
  return dt == MMF_BF16 ? launch_t<bf16>(a, g, stream) : launch_t<float>(a, g, stream);
}

}  // namespace mmf
