// Prefill token mixer in one kernel: the f|c|g ternary contraction on the
// tcgen05 tensor cores with the MLGRU gates and recurrence in its epilogue.
//
// "MatMul-free language models" (DataCamp blog), section "Core components:
// MLGRU and GLU", and the hysenlabs review, section "HGRN attention": the
// token mixer projects the input with three BitLinears and runs a gated
// recurrence over the tokens. Per channel:
//   f = sigmoid(f~), c = SiLU(c~), g = sigmoid(g~)
//   h_t = f h_{t-1} + (1 - f) c,   o'_t = g h_t
// The pre-activations f~, c~, g~ exist only in tensor memory and registers
// (rounded to the activation type exactly where a separate contraction would
// have stored them); the kernel writes o' and the final state, nothing else.
//
// Tile: 128 tokens x 64 channels x the three gates (MMA N = 192: rows of the
// f, c and g weight matrices for the same 64 channels), K in 128-byte steps.
// Main loop as in the plain contraction (tgemm_tc.cu): persistent CTAs, warp 0
// TMA (activation tile + three 64-row packed weight boxes), warp 1 TMEM and the
// single MMA thread, warps 10-13 unpack the 2-bit codes into the UMMA layout,
// double-buffered accumulators.
// Epilogue (warps 2-9; warp w reads TMEM lanes 32(w%4).., i.e. 32 tokens, and
// one half of the 64 channels): each thread owns one token.
//   1. rescale f~, c~ (rounded to the storage type), gates, b = (1-f) c; an
//      inclusive warp-shuffle scan of the affine maps h -> f h + b over its 32
//      tokens; the last lane records the quarter's map in shared memory.
//   2. one warp folds the four quarter maps into the tile's map, publishes it
//      at once (aggregate), looks back over the previous 128-token tiles of
//      the same channels (a published leaving state ends the walk, an
//      aggregate is composed in; the sequence's first tile starts from the
//      state h), publishes the tile's leaving state and the state entering
//      each quarter.
//   3. every thread applies its prefix map to its quarter's entering state,
//      multiplies by g and stores o' through a swizzled staging box and a TMA
//      tensor store.
// Publication is fence-free (one 64-bit word per value pair, scratch filled
// with an all-ones NaN pattern beforehand). Tile order is chunk-major: all
// sequences' first 128 tokens, then the next 128, ... (channels fastest), so a
// tile's predecessor (same channels, previous 128 tokens) is a whole chunk of
// tiles earlier and normally already done. CTAs take tiles in increasing index
// order and every wait is on a smaller index, so the smallest unfinished tile
// can always proceed; every wait is bounded (status word, no trap).
#include "kernels.cuh"
#include "umma.cuh"

namespace mmf {

namespace {

constexpr int BM = 128, CH = 64, BN = 3 * CH, BK = 128;
constexpr int NS = 4;                      // TMA ring
constexpr int NB = 2;                      // unpacked-code ring
constexpr int A_BYTES = BM * BK;           // 16 KiB activation codes
constexpr int BP_BYTES = BN * BK / 4;      // 6 KiB packed codes (3 boxes of 64 rows)
constexpr int BU_BYTES = BN * BK;          // 24 KiB unpacked codes
constexpr int kEpiWarps = 8, kEpiWarp0 = 2, kUnpackWarp0 = kEpiWarp0 + kEpiWarps;
constexpr int kUnpackThreads = 128;
constexpr int kThreads = (kUnpackWarp0 + kUnpackThreads / 32) * 32;   // 14 warps
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccStride = 256;       // TMEM columns between the two accumulators
constexpr int kWordsPerTile = 96;          // 64 aggregate words (one per channel) + 32 leaving-state words
constexpr uint32_t kUnset = 0xffffffffu;

template <int OB>
struct __align__(1024) MlgruSmem {
  static constexpr int kStageBytes = 32 * 32 * OB;
  uint8_t a[NS][A_BYTES];
  uint8_t bu[NB][BU_BYTES];
  uint8_t stage[kEpiWarps][2][kStageBytes];
  uint32_t bp[NS][BP_BYTES / 4];
  float2 qmap[4][CH];                      // map of each 32-token quarter, per channel
  float hq[4][CH];                         // state entering each quarter
  uint64_t tma_full[NS];
  uint64_t tma_empty[NS];
  uint64_t bu_full[NB];
  uint64_t bu_empty[NB];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr uint32_t kIdesc = umma_idesc_i8(BM, BN);

struct MlgruArgs {
  TGemmArgs g;          // w/gamma/bias of f, c, g; q, s, qsum; M; out = o' [M, d]
  int T, d;             // sequence length (multiple of BM), channels (multiple of CH)
  int nseq;             // sequences B = M / T
  int m_tiles, n_tiles;
  float* h;             // [B, d] fp32 state, read at each sequence's first tile, written at its last
  float2* rec;          // kWordsPerTile words per tile, all-ones before the launch
  int* status;
};

// Tile index -> (token tile, channel tile); chunk-major: index = (j * B + b) *
// n_tiles + nt for chunk j of sequence b, so token tile mt = b * (T / BM) + j.
__device__ __forceinline__ void tile_coords(const MlgruArgs& p, int tile, int& mt, int& nt, int& b, int& j) {
  const int per_chunk = p.nseq * p.n_tiles;
  j = tile / per_chunk;
  const int rem = tile - j * per_chunk;
  b = rem / p.n_tiles;
  nt = rem - b * p.n_tiles;
  mt = b * (p.T / BM) + j;
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Named barrier of the epilogue warps; returns whether any of them passed true.
__device__ __forceinline__ bool epi_bar_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " barrier.cta.red.or.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kEpiThreads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void epi_bar() { asm volatile("barrier.cta.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); }

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

// f = sigmoid(zf), b = (1 - f) SiLU(zc), one reciprocal for both logistic
// terms; exponents capped at 40 so the product stays finite (below -40 the
// logistic is under 5e-18 and the cap moves it by less than that).
__device__ __forceinline__ void gate_fb(float zf, float zc, float& f, float& b) {
  const float pf = 1.0f + ex2_approx(fminf(-zf * kLog2e, kMaxExp2));
  const float pc = 1.0f + ex2_approx(fminf(-zc * kLog2e, kMaxExp2));
  const float r = rcp_approx(pf * pc);
  f = pc * r;
  b = (1.0f - f) * (zc * (pf * r));
}
__device__ __forceinline__ float sigmoid_fast(float z) { return rcp_approx(1.0f + ex2_approx(-z * kLog2e)); }

// Stage 16 of the 32 columns (half k) of row r of a 32 x 32 output box in the
// layout the output map's swizzle expects: 2-byte types 64-byte rows with the
// 64B swizzle (16-byte chunk c at c ^ ((r>>1)&3)), 4-byte types 128-byte rows
// with the 128B swizzle (chunk c at c ^ (r&7)).
__device__ __forceinline__ void stage_half(uint8_t* buf, int r, int k, const float (&v)[16], bf16*) {
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int c = 2 * k + cc;
    uint4 u;
    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h2[i] = __floats2bfloat162_rn(v[8 * cc + 2 * i], v[8 * cc + 2 * i + 1]);
    *reinterpret_cast<uint4*>(buf + r * 64 + ((c ^ ((r >> 1) & 3)) << 4)) = u;
  }
}
__device__ __forceinline__ void stage_half(uint8_t* buf, int r, int k, const float (&v)[16], float*) {
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int c = 4 * k + cc;
    *reinterpret_cast<float4*>(buf + r * 128 + ((c ^ (r & 7)) << 4)) =
        make_float4(v[4 * cc], v[4 * cc + 1], v[4 * cc + 2], v[4 * cc + 3]);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    tgemm_tc_mlgru_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_f,
                          const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_g,
                          const __grid_constant__ CUtensorMap map_out, const MlgruArgs p) {
  constexpr int OB = (int)sizeof(T);
  using Smem = MlgruSmem<OB>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;
  const int n_tiles_total = p.m_tiles * p.n_tiles;
  const int nk = ceil_div(p.g.K, BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.tma_full[s], 1);
      mbar_init(&sm.tma_empty[s], 1);
    }
    for (int u = 0; u < NB; ++u) {
      mbar_init(&sm.bu_full[u], kUnpackThreads);
      mbar_init(&sm.bu_empty[u], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.tmem_full[a], 1);
      mbar_init(&sm.tmem_empty[a], kEpiThreads);
    }
    mbar_init(&sm.mma_drain, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&map_a);
    prefetch_tmap(&map_out);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;
  pdl_trigger();
  pdl_wait();   // codes, scales and the state are the predecessors' outputs

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const CUtensorMap* maps[3] = {&map_f, &map_c, &map_g};
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x) {
        int mt, nt, b, j;
        tile_coords(p, tile, mt, nt, b, j);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % NS;
          if (!mbar_wait(&sm.tma_empty[s], ((it / NS) & 1) ^ 1, abort_flag, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&sm.tma_full[s], A_BYTES + BP_BYTES);
          tma_load_2d(sm.a[s], &map_a, kb * BK, mt * BM, &sm.tma_full[s]);
          for (int gsel = 0; gsel < 3; ++gsel)
            tma_load_2d(&sm.bp[s][gsel * CH * (BK / 16)], maps[gsel], kb * (BK / 16), nt * CH, &sm.tma_full[s]);
        }
      }
      for (uint32_t j = (it > NS ? it - NS : 0); j < it; ++j)
        mbar_wait(&sm.tma_full[j % NS], (j / NS) & 1, abort_flag, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tl = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x, ++tl) {
        const int acc = tl & 1;
        const uint32_t acc_ph = (tl >> 1) & 1;
        if (!mbar_wait(&sm.tmem_empty[acc], acc_ph ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccStride;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % NS, u = it % NB;
          if (!mbar_wait(&sm.bu_full[u], (it / NB) & 1, abort_flag, p.status) ||
              !mbar_wait(&sm.tma_full[s], (it / NS) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = umma_desc_sw128(smem_u32(sm.a[s]));
          const uint64_t bdesc = umma_desc_sw128(smem_u32(sm.bu[u]));
#pragma unroll
          for (int j = 0; j < BK / 32; ++j)
            umma_i8(d_tmem, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), kIdesc, (kb | j) != 0);
          umma_commit(&sm.tma_empty[s]);
          umma_commit(&sm.bu_empty[u]);
        }
        if (ok) umma_commit(&sm.tmem_full[acc]);
      }
      umma_commit(&sm.mma_drain);
      mbar_wait(&sm.mma_drain, 0, abort_flag, nullptr);
    }
  } else if (warp >= kUnpackWarp0) {
    // ------------------------------------------------------------ unpack 2-bit codes to int8
    // 384 (row, half-row) units per K-step: unit id = tid + 128 i reads the 16
    // bytes at id * 16 of the packed tile (row id/2, columns 64 (id%2) ..+63)
    const int tid = threadIdx.x - kUnpackWarp0 * 32;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x) {
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % NS, u = it % NB;
        if (!mbar_wait(&sm.tma_full[s], (it / NS) & 1, abort_flag, p.status) ||
            !mbar_wait(&sm.bu_empty[u], ((it / NB) & 1) ^ 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        const uint4* src = reinterpret_cast<const uint4*>(sm.bp[s]);
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const int id = tid + kUnpackThreads * i;
          const int n = id >> 1, hh = id & 1;
          const uint4 w4 = src[id];
          const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
          uint8_t* dst = sm.bu[u] + n * BK;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * hh + e;
            const uint32_t w = ws[e];
            uint4 v;
            v.x = w & 0x03030303u;
            v.y = (w >> 2) & 0x03030303u;
            v.z = (w >> 4) & 0x03030303u;
            v.w = (w >> 6) & 0x03030303u;
            *reinterpret_cast<uint4*>(dst + ((c ^ (n & 7)) << 4)) = v;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&sm.bu_full[u]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue: gates + recurrence (8 warps)
    const int ew = warp - kEpiWarp0;
    const int quarter = warp & 3;                 // tokens 32*quarter .. +31 of the tile
    const int half = ew >> 2;                     // channels 32*half .. +31 of the tile
    const int tok = quarter * 32 + lane;
    uint8_t* stage0 = sm.stage[ew][0];
    uint8_t* stage1 = sm.stage[ew][1];
    int nst = 0;
    uint32_t tl = 0;
    const int chunks = p.T / BM;                  // token tiles per sequence
    for (int tile = blockIdx.x; tile < n_tiles_total; tile += gridDim.x, ++tl) {
      int mt, nt, b, j;
      tile_coords(p, tile, mt, nt, b, j);
      const int acc = tl & 1;
      const uint32_t acc_ph = (tl >> 1) & 1;
      const bool got = mbar_wait(&sm.tmem_full[acc], acc_ph, abort_flag, p.status);
      if (epi_bar_or(!got)) break;                // all eight warps leave together
      tc_fence_after();
      const int m = mt * BM + tok;
      const int c0 = nt * CH;
      const float inv_s = 1.0f / p.g.s[m];
      const int qs = p.g.qsum[m];
      const float sc_f = *p.g.gamma[0] * inv_s, sc_c = *p.g.gamma[1] * inv_s, sc_g = *p.g.gamma[2] * inv_s;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * kAccStride;

      // 1. gates, inclusive scan of this quarter's maps per channel
      float A[32], Bv[32];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        uint32_t rf[16], rc[16];
        tmem_ld16(tbase + half * 32 + 16 * k, rf);
        tmem_ld16(tbase + CH + half * 32 + 16 * k, rc);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int ch = c0 + half * 32 + 16 * k + i;
          float zf = (float)((int)rf[i] - qs) * sc_f;
          float zc = (float)((int)rc[i] - qs) * sc_c;
          if (p.g.bias[0] != nullptr) zf += p.g.bias[0][ch];
          if (p.g.bias[1] != nullptr) zc += p.g.bias[1][ch];
          float f, bb;
          gate_fb(round_to<T>(zf), round_to<T>(zc), f, bb);   // the pre-activations' storage point
          float a = f, v = bb;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float ap = __shfl_up_sync(0xffffffffu, a, o);
            const float vp = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) {
              v = fmaf(a, vp, v);
              a *= ap;
            }
          }
          A[16 * k + i] = a;
          Bv[16 * k + i] = v;
          if (lane == 31) sm.qmap[quarter][half * 32 + 16 * k + i] = make_float2(a, v);
        }
      }
      epi_bar();

      // 2. tile map, aggregate, look-back, leaving state, quarter entering states
      if (ew == 0) {
        float2* mine = p.rec + (size_t)tile * kWordsPerTile;
        float2 qa[4], qb[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 m0 = sm.qmap[q][2 * lane], m1 = sm.qmap[q][2 * lane + 1];
          qa[q] = make_float2(m0.x, m1.x);
          qb[q] = make_float2(m0.y, m1.y);
        }
        float2 ta = make_float2(1.0f, 1.0f), tb = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          tb = make_float2(fmaf(qa[q].x, tb.x, qb[q].x), fmaf(qa[q].y, tb.y, qb[q].y));
          ta = make_float2(qa[q].x * ta.x, qa[q].y * ta.y);
        }
        float2 hv = make_float2(0.0f, 0.0f);
        if (j == 0) {
          hv = *reinterpret_cast<const float2*>(p.h + (size_t)b * p.d + c0 + 2 * lane);
        } else {
          st_word(mine + 2 * lane, make_float2(ta.x, tb.x));
          st_word(mine + 2 * lane + 1, make_float2(ta.y, tb.y));
          float2 acc_a = make_float2(1.0f, 1.0f), acc_b = make_float2(0.0f, 0.0f);
          int prev = tile - p.nseq * p.n_tiles;      // same channels, previous 128 tokens
          const long long t_start = clock64();
          while (true) {
            const float2* theirs = p.rec + (size_t)prev * kWordsPerTile;
            const float2 hp = ld_word(theirs + 64 + lane);
            const float2 w0 = ld_word(theirs + 2 * lane), w1 = ld_word(theirs + 2 * lane + 1);
            if (is_set(hp)) {
              hv = make_float2(fmaf(acc_a.x, hp.x, acc_b.x), fmaf(acc_a.y, hp.y, acc_b.y));
              break;
            }
            if (is_set(w0) && is_set(w1)) {          // aggregate only: compose it, look one tile further
              acc_b = make_float2(fmaf(acc_a.x, w0.y, acc_b.x), fmaf(acc_a.y, w1.y, acc_b.y));
              acc_a = make_float2(acc_a.x * w0.x, acc_a.y * w1.x);
              prev -= p.nseq * p.n_tiles;            // the sequence's first tile always publishes its state
              continue;
            }
            if (clock64() - t_start > kWaitCycles) { // give up: continue from zero (reported)
              if (p.status) atomicExch(p.status, 2);
              break;
            }
          }
        }
        const float2 hout = make_float2(fmaf(ta.x, hv.x, tb.x), fmaf(ta.y, hv.y, tb.y));
        st_word(mine + 64 + lane, hout);
        if (j == chunks - 1) *reinterpret_cast<float2*>(p.h + (size_t)b * p.d + c0 + 2 * lane) = hout;
        float2 e = hv;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          sm.hq[q][2 * lane] = e.x;
          sm.hq[q][2 * lane + 1] = e.y;
          e = make_float2(fmaf(qa[q].x, e.x, qb[q].x), fmaf(qa[q].y, e.y, qb[q].y));
        }
      }
      epi_bar();

      // 3. o' = g * (prefix map applied to the quarter's entering state),
      //    staged 16 channels at a time
      if (lane == 0 && nst >= 2) bulk_wait_read_le1();   // the store that last used this buffer has read it
      __syncwarp();
      uint8_t* buf = (nst & 1) ? stage1 : stage0;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        uint32_t rg[16];
        tmem_ld16(tbase + 2 * CH + half * 32 + 16 * k, rg);
        float out[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int cl = half * 32 + 16 * k + i;
          float zg = (float)((int)rg[i] - qs) * sc_g;
          if (p.g.bias[2] != nullptr) zg += p.g.bias[2][c0 + cl];
          const float hcur = fmaf(A[16 * k + i], sm.hq[quarter][cl], Bv[16 * k + i]);
          out[i] = sigmoid_fast(round_to<T>(zg)) * hcur;
        }
        stage_half(buf, lane, k, out, (T*)nullptr);
      }
      tc_fence_before();
      mbar_arrive(&sm.tmem_empty[acc]);           // accumulator read completely
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tma_store_2d(&map_out, buf, c0 + half * 32, mt * BM + quarter * 32);
      ++nst;
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

template <typename T>
cudaError_t launch_typed(const CUtensorMap& ma, const CUtensorMap (&mw)[3], const MlgruArgs& p, cudaStream_t stream) {
  CUtensorMap mo;
  const int esize = (int)sizeof(T);
  const CUtensorMapDataType odt = esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const CUtensorMapSwizzle oswz = esize == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tma_2d(&mo, p.g.out, odt, esize, (uint64_t)p.d, (uint64_t)p.g.M, 32, 32, oswz))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(MlgruSmem<sizeof(T)>) + 1024;
  auto kern = tgemm_tc_mlgru_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = std::min(tiles, num_sms());
  return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, stream, ma, mw[0], mw[1], mw[2], mo, p);
}

}  // namespace

bool tgemm_tc_mlgru_supported(const TGemmArgs& a, int T, int d) {
  return a.nseg == 3 && a.N == d && T > 0 && T % BM == 0 && d % CH == 0 && a.M % T == 0 && a.K % 64 == 0 &&
         tma_available();
}

size_t tgemm_tc_mlgru_ws_bytes(int B, int T, int d) {
  return 256 + sizeof(float2) * kWordsPerTile * (size_t)ceil_div(T, BM) * B * ceil_div(d, CH);
}

cudaError_t reset_tgemm_tc_mlgru_ws(void* ws, int B, int T, int d, cudaStream_t stream) {
  return cudaMemsetAsync(ws, 0xff, tgemm_tc_mlgru_ws_bytes(B, T, d), stream);
}

cudaError_t launch_tgemm_tc_mlgru(const TGemmArgs& a, mmf_dtype dt, int T, int d, float* h, void* ws, int* status,
                                  cudaStream_t stream) {
  if (a.M == 0) return cudaSuccess;
  if (!tgemm_tc_mlgru_supported(a, T, d)) return cudaErrorNotSupported;
  CUtensorMap ma, mw[3];
  if (!make_tma_2d(&ma, a.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.K, (uint64_t)a.M, BK, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  for (int r = 0; r < 3; ++r)
    if (!make_tma_2d(&mw[r], a.w[r], CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)(a.K / 16), (uint64_t)d, BK / 16,
                     CH, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  MlgruArgs p;
  p.g = a;
  p.T = T;
  p.d = d;
  p.nseq = a.M / T;
  p.m_tiles = a.M / BM;
  p.n_tiles = d / CH;
  p.h = h;
  p.rec = reinterpret_cast<float2*>(static_cast<char*>(ws) + 256);
  p.status = status;
  return dt == MMF_BF16 ? launch_typed<bf16>(ma, mw, p, stream) : launch_typed<float>(ma, mw, p, stream);
}

}  // namespace mmf
