// Prefill ternary contraction on the 5th-generation tensor cores (tcgen05,
// kind::i8, accumulators in tensor memory).
//
// "MatMul-free language models" (DataCamp blog), section "Replacing MatMul
// with ternary operations": with weights in {-1,0,1} the contraction is exact
// integer add/subtract work, so an int8 x int8 -> int32 tensor-core product of
// the activation codes with the ternary codes gives the exact accumulators.
// The stored weight code is w + 1 (unsigned byte 0..2); the kernel computes
// sum_k q[m,k] (w[n,k] + 1) with an s8 x u8 MMA and the epilogue subtracts the
// token's code sum: acc = raw - sum_k q[m,k].
//
// Tile: 128 tokens (M) x 256 output columns (N) x 128 k-bytes per K-step.
// Persistent CTAs (one per SM, 320 threads), warp-specialised:
//   warp 0      TMA producer: int8 activation tile (128B-swizzled, the UMMA
//               K-major SW128 layout) + 2-bit packed weight tile, 4-deep ring
//   warp 1      TMEM owner + single-thread MMA issuer (4 x K=32 per K-step)
//   warps 2..5  epilogue: tcgen05.ld of the int32 accumulators, rescale
//               (+bias, +residual, SiLU*up), swizzled staging in shared
//               memory, TMA tensor store (coalesced, clipped at the M edge)
//   warps 6..9  unpack: packed 2-bit codes -> int8 bytes written directly in
//               the SW128 K-major layout the MMA reads, 2-deep ring
// Two TMEM accumulators (2 x 256 columns) let the epilogue of one tile overlap
// the main loop of the next. Variant RB (bf16 outputs with a residual, short
// K): each epilogue warp loads the whole residual of its half tile into four
// staging buffers before the tile's accumulator is ready, instead of one 32 x
// 32 box at a time on the critical path.
// Variant UNP: when the codes are also held one byte per weight in HBM (a
// block keeps such a copy for prefill), the producer TMA-loads the weight tile
// straight into the SW128 layout next to the activation tile (3-stage ring of
// 16 + 32 KiB) and the unpack warps stay idle; unpacking 32 KiB per k-step
// through shared memory was the largest cost of the main loop. Every mbarrier wait is bounded: on timeout the
// kernel records an error in the status word, raises a CTA-wide abort flag,
// and all roles leave their loops; nothing traps.
#include "kernels.cuh"
#include "umma.cuh"

namespace mmf {

namespace {

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int NB = 2;                     // unpacked-code ring depth
constexpr int A_BYTES = BM * BK;          // 16 KiB int8 activations
constexpr int BP_BYTES = BN * BK / 4;     // 8 KiB packed codes (2 bit)
constexpr int BU_BYTES = BN * BK;         // 32 KiB unpacked codes (int8)
constexpr int HALF = BN / 2;              // rows per weight TMA box
constexpr int kEpiWarps = 8;              // two per TMEM lane quarter, splitting the columns
constexpr int kEpiWarp0 = 2, kUnpackWarp0 = kEpiWarp0 + kEpiWarps;
constexpr int kUnpackThreads = 128;
constexpr int kThreads = (kUnpackWarp0 + kUnpackThreads / 32) * 32;   // 14 warps
constexpr int kEpiChunk = 32;             // output columns per TMA store box (x 32 rows)
constexpr uint32_t kTmemCols = 512;

// Shared memory; OB = bytes of one output element (2: bf16, 4: fp32 / int32).
// The TMA ring is 4 deep for 2-byte outputs and 3 deep for 4-byte outputs,
// whose staging boxes are twice as large; with UNP (a weight tile per stage)
// also 4 deep for 2-byte outputs (225 KB of the 227 KB) and 3 for 4-byte ones.
// RB (residual prefetch, 2-byte outputs only): the ring is 3 deep and each
// epilogue warp has 4 staging buffers, one per 32-column chunk of its half
// tile, into which the whole tile's residual is loaded before the tile's
// accumulator is ready.
template <int OB, bool UNP, bool RB = false>
struct __align__(1024) SmemLayout {
  static constexpr int NS = RB ? 3 : (UNP ? (OB == 2 ? 4 : 3) : (OB == 2 ? 4 : 3));
  static constexpr int NSTG = RB ? HALF / kEpiChunk : 2;   // staging buffers per epilogue warp
  static constexpr int NBU = UNP ? NS : NB;        // int8 weight tiles: per TMA stage (UNP) or unpack ring
  static constexpr int NBP = UNP ? 1 : NS;         // packed weight tiles (unused with UNP)
  static constexpr int kStageBytes = 32 * kEpiChunk * OB;
  uint8_t a[NS][A_BYTES];                          // 1024-aligned: SW128 atoms
  uint8_t bu[NBU][BU_BYTES];                       // 1024-aligned: SW128 atoms
  uint8_t stage[kEpiWarps][NSTG][kStageBytes];     // epilogue staging (1024-aligned)
  uint32_t bp[NBP][UNP ? 4 : BP_BYTES / 4];
  uint64_t tma_full[NS];
  uint64_t tma_empty[NS];
  uint64_t bu_full[NB];
  uint64_t bu_empty[NB];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t res_full[kEpiWarps][NSTG];              // residual box landed in a staging buffer
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr uint32_t kIdesc = umma_idesc_i8(BM, BN);

// ---------------------------------------------------------------- tile geometry
struct TcArgs {
  TGemmArgs g;
  int m_tiles, n_tiles;
  int* status;
  long long wait_cycles;   // bound of every wait
  uint32_t skip_it;        // test hook: CTA 0 never loads this k-step (~0u: none)
};

// Rows of weight segment `seg` starting at `row0` feed half `h` of tile `nt`.
__device__ __forceinline__ void half_source(const TcArgs& p, Epi epi, int nt, int h, int& seg, int& row0) {
  if (epi == Epi::kGlu) {
    seg = h;
    row0 = nt * HALF;
  } else {
    const int gcol = nt * BN + h * HALF;
    const int total = p.g.nseg * p.g.N;
    if (gcol >= total) {   // past the last segment: a fully out-of-bounds box reads zeros
      seg = p.g.nseg - 1;
      row0 = p.g.N;
    } else {
      seg = gcol / p.g.N;
      row0 = gcol % p.g.N;
    }
  }
}

template <Epi EPI, typename T, bool UNP, bool RB = false>
__global__ void __launch_bounds__(kThreads, 1)
    tgemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b0,
                    const __grid_constant__ CUtensorMap map_b1, const __grid_constant__ CUtensorMap map_b2,
                    const __grid_constant__ CUtensorMap map_out, const __grid_constant__ CUtensorMap map_res,
                    const TcArgs p) {
  constexpr int OB = EPI == Epi::kAcc ? 4 : (int)sizeof(T);
  static_assert(!RB || (EPI == Epi::kStore && OB == 2), "residual prefetch: kStore with 2-byte outputs");
  using Smem = SmemLayout<OB, UNP, RB>;
  constexpr int NS = Smem::NS;
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
      mbar_init(&sm.tmem_empty[a], kEpiWarps * 32);
    }
    for (int w = 0; w < kEpiWarps; ++w)
      for (int c = 0; c < Smem::NSTG; ++c) mbar_init(&sm.res_full[w][c], 1);
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
  // programmatic dependent launch: the set-up above overlaps the predecessor's
  // tail; its outputs (codes, scales, residual) are read only after this
  pdl_trigger();
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const CUtensorMap* maps[3] = {&map_b0, &map_b1, &map_b2};
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x) {
        const int mt = tile / p.n_tiles, nt = tile % p.n_tiles;
        int seg0, row0, seg1, row1;
        half_source(p, EPI, nt, 0, seg0, row0);
        half_source(p, EPI, nt, 1, seg1, row1);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % NS;
          if (!mbar_wait(&sm.tma_empty[s], ((it / NS) & 1) ^ 1, abort_flag, p.status, p.wait_cycles)) { ok = false; break; }
          if (it == p.skip_it && blockIdx.x == 0) continue;   // test hook: these copies are never issued
          if constexpr (UNP) {   // int8 weight rows straight into the SW128 tile of this stage
            mbar_arrive_expect_tx(&sm.tma_full[s], A_BYTES + BU_BYTES);
            tma_load_2d(sm.a[s], &map_a, kb * BK, mt * BM, &sm.tma_full[s]);
            tma_load_2d(sm.bu[s], maps[seg0], kb * BK, row0, &sm.tma_full[s]);
            tma_load_2d(sm.bu[s] + HALF * BK, maps[seg1], kb * BK, row1, &sm.tma_full[s]);
          } else {
            mbar_arrive_expect_tx(&sm.tma_full[s], A_BYTES + BP_BYTES);
            tma_load_2d(sm.a[s], &map_a, kb * BK, mt * BM, &sm.tma_full[s]);
            tma_load_2d(&sm.bp[s][0], maps[seg0], kb * (BK / 16), row0, &sm.tma_full[s]);
            tma_load_2d(&sm.bp[s][HALF * (BK / 16)], maps[seg1], kb * (BK / 16), row1, &sm.tma_full[s]);
          }
        }
      }
      // let every copy this thread issued land before the CTA can exit
      for (uint32_t j = (it > NS ? it - NS : 0); j < it; ++j)
        if (j != p.skip_it || blockIdx.x != 0) mbar_drain(&sm.tma_full[j % NS], (j / NS) & 1, p.wait_cycles);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tl = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x, ++tl) {
        const int acc = tl & 1;
        const uint32_t acc_ph = (tl >> 1) & 1;
        if (!mbar_wait(&sm.tmem_empty[acc], acc_ph ^ 1, abort_flag, p.status, p.wait_cycles)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % NS, u = UNP ? s : (int)(it % NB);
          if ((!UNP && !mbar_wait(&sm.bu_full[u], (it / NB) & 1, abort_flag, p.status, p.wait_cycles)) ||
              !mbar_wait(&sm.tma_full[s], (it / NS) & 1, abort_flag, p.status, p.wait_cycles)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = umma_desc_sw128(smem_u32(sm.a[s]));
          const uint64_t bdesc = umma_desc_sw128(smem_u32(sm.bu[u]));
#pragma unroll
          for (int j = 0; j < BK / 32; ++j)   // advance 32 bytes of K inside the swizzle atom
            umma_i8(d_tmem, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), kIdesc, (kb | j) != 0);
          umma_commit(&sm.tma_empty[s]);
          if constexpr (!UNP) umma_commit(&sm.bu_empty[u]);
        }
        if (ok) umma_commit(&sm.tmem_full[acc]);
      }
      // every MMA this thread issued has finished before TMEM can be released
      umma_commit(&sm.mma_drain);
      mbar_drain(&sm.mma_drain, 0, p.wait_cycles);
    }
  } else if (warp >= kUnpackWarp0) {
    // ------------------------------------------------------------ unpack 2-bit codes to int8 (idle with UNP)
    if constexpr (!UNP) {
    // 512 (row, half-row) units per K-step; unit id = tid + 128 i reads the 16
    // bytes at id * 16 of the packed tile (row id/2, columns 64 (id%2) ..+63),
    // so each warp reads 512 contiguous bytes; writes land in distinct banks.
    const int tid = threadIdx.x - kUnpackWarp0 * 32;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x) {
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % NS, u = it % NB;
        if (!mbar_wait(&sm.tma_full[s], (it / NS) & 1, abort_flag, p.status, p.wait_cycles) ||
            !mbar_wait(&sm.bu_empty[u], ((it / NB) & 1) ^ 1, abort_flag, p.status, p.wait_cycles)) {
          ok = false;
          break;
        }
        const uint4* src = reinterpret_cast<const uint4*>(sm.bp[s]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int id = tid + kUnpackThreads * i;
          const int n = id >> 1, h = id & 1;
          const uint4 w4 = src[id];
          const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
          uint8_t* dst = sm.bu[u] + n * BK;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * h + e;         // 16-column chunk of this row
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
    }
  } else {
    // ------------------------------------------------------------ epilogue (8 warps)
    const int ew = warp - kEpiWarp0;              // 0..7
    const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
    const int group = ew >> 2;                    // which half of the columns this warp takes
    const int row_in_tile = quarter * 32 + lane;
    uint8_t* stage0 = sm.stage[ew][0];
    uint8_t* stage1 = sm.stage[ew][1];
    int nst = 0;                                  // boxes stored by this warp so far
    uint32_t nres = 0;                            // residual boxes loaded by this warp so far
    uint32_t tl = 0;
    const bool has_res = EPI == Epi::kStore && p.g.residual != nullptr;
    // Wait until the store that last used staging buffer (nst & 1) has read it.
    auto claim = [&](uint8_t*& buf) {
      if (lane == 0 && nst >= 2) bulk_wait_read_le1();
      __syncwarp();
      buf = (nst & 1) ? stage1 : stage0;
    };
    auto release = [&](int x, int y, uint8_t* buf) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tma_store_2d(&map_out, buf, x, y);
      ++nst;
    };
    bool alive = true;
    uint32_t res_pending = 0;                     // RB: this tile's residual boxes not yet waited on
    for (int tile = blockIdx.x; tile < n_tiles_total && alive; tile += gridDim.x, ++tl) {
      const int mt = tile / p.n_tiles, nt = tile % p.n_tiles;
      const int acc = tl & 1;
      const uint32_t acc_ph = (tl >> 1) & 1;
      if constexpr (RB) {   // the whole half tile's residual, before the accumulator is ready
        int seg, row0;
        half_source(p, EPI, nt, group, seg, row0);
        if (nt * BN + group * HALF < p.g.N) {
          if (lane == 0) {
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");   // last tile's stores have read them
            for (int c = 0; c < Smem::NSTG; ++c) {
              mbar_arrive_expect_tx(&sm.res_full[ew][c], 32 * kEpiChunk * OB);
              tma_load_2d(sm.stage[ew][c], &map_res, row0 + 32 * c, mt * BM + quarter * 32, &sm.res_full[ew][c]);
            }
          }
          res_pending = (1u << Smem::NSTG) - 1;
        }
      }
      const bool got = mbar_wait(&sm.tmem_full[acc], acc_ph, abort_flag, p.status, p.wait_cycles);
      __syncwarp();                               // tcgen05.ld below is warp-collective
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int m = mt * BM + row_in_tile;
      const int y0 = mt * BM + quarter * 32;
      const bool row_ok = m < p.g.M;
      const float inv_s = row_ok ? 1.0f / p.g.s[m] : 0.0f;
      const int qs = row_ok ? p.g.qsum[m] : 0;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      if constexpr (EPI == Epi::kGlu) {
        const float sc_u = *p.g.gamma[0] * inv_s, sc_v = *p.g.gamma[1] * inv_s;
        for (int cc = 0; cc < 2; ++cc) {
          const int c = group * 2 + cc;           // 32-column chunk of the gate / up halves
          uint32_t ru[32], rv[32];
          tmem_ld32(tbase + 32 * c, ru);
          tmem_ld32(tbase + HALF + 32 * c, rv);
          const int n0 = nt * HALF + 32 * c;
          float out[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float uu = (float)((int)ru[j] - qs) * sc_u;
            float vv = (float)((int)rv[j] - qs) * sc_v;
            if (p.g.bias[0] != nullptr) uu += p.g.bias[0][n0 + j];
            if (p.g.bias[1] != nullptr) vv += p.g.bias[1][n0 + j];
            out[j] = silu_fast(uu) * vv;
          }
          uint8_t* buf;
          claim(buf);
          stage_row(buf, lane, out, (T*)nullptr);
          release(n0, y0, buf);
        }
      } else {
        const int h = group;                      // 128-column half of the tile
        int seg, row0;
        half_source(p, EPI, nt, h, seg, row0);
        if (RB && nt * BN + h * HALF < p.g.N) {   // residual already on its way into stage[ew][c]
          const float sc = *p.g.gamma[0] * inv_s;
          const float* bias = p.g.bias[0];
          for (int c = 0; c < Smem::NSTG; ++c) {
            const int n0 = row0 + 32 * c;
            uint8_t* buf = sm.stage[ew][c];
            uint32_t r[32];
            tmem_ld32(tbase + h * HALF + 32 * c, r);
            float out[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              float v = (float)((int)r[j] - qs) * sc;
              if (bias != nullptr) v += bias[n0 + j];
              out[j] = v;
            }
            const bool ok = mbar_wait(&sm.res_full[ew][c], nres & 1, abort_flag, p.status, p.wait_cycles);
            if (!__all_sync(0xffffffffu, ok)) { alive = false; break; }
            res_pending &= ~(1u << c);
            add_staged_row(buf, lane, out, (T*)nullptr);
            __syncwarp();                         // every row read before any row is overwritten
            stage_row(buf, lane, out, (T*)nullptr);
            release(n0, y0, buf);
          }
          ++nres;
        } else if (!RB && nt * BN + h * HALF < p.g.nseg * p.g.N) {
          const float sc = *p.g.gamma[seg] * inv_s;
          const float* bias = p.g.bias[seg];
          for (int c = 0; c < HALF / kEpiChunk; ++c) {
            const int n0 = row0 + 32 * c;
            const int x0 = seg * p.g.N + n0;
            uint8_t* buf;
            claim(buf);
            if (has_res && lane == 0) {           // residual box -> this staging buffer
              mbar_arrive_expect_tx(&sm.res_full[ew][0], 32 * kEpiChunk * OB);
              tma_load_2d(buf, &map_res, n0, y0, &sm.res_full[ew][0]);
            }
            uint32_t r[32];
            tmem_ld32(tbase + h * HALF + 32 * c, r);
            if constexpr (EPI == Epi::kAcc) {
              stage_row_i32(buf, lane, r, qs);
            } else {
              float out[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                float v = (float)((int)r[j] - qs) * sc;
                if (bias != nullptr) v += bias[n0 + j];
                out[j] = v;
              }
              if (has_res) {
                const bool ok = mbar_wait(&sm.res_full[ew][0], nres & 1, abort_flag, p.status, p.wait_cycles);
                ++nres;
                if (!__all_sync(0xffffffffu, ok)) { alive = false; break; }
                add_staged_row(buf, lane, out, (T*)nullptr);
                __syncwarp();                     // every row read before any row is overwritten
              }
              stage_row(buf, lane, out, (T*)nullptr);
            }
            release(x0, y0, buf);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.tmem_empty[acc]);
    }
    if constexpr (RB) {   // residual boxes issued for a tile that was given up: let them land (bounded)
      if (lane == 0)
        for (int c = 0; c < Smem::NSTG; ++c)
          if (res_pending & (1u << c)) mbar_drain(&sm.res_full[ew][c], nres & 1, p.wait_cycles);
    }
    if (lane == 0) bulk_wait_all();   // stores complete before the CTA exits
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

// ---------------------------------------------------------------- host side
template <Epi EPI, typename T, bool UNP, bool RB = false>
cudaError_t launch_typed(const CUtensorMap& ma, const CUtensorMap (&mb)[3], const TcArgs& p, cudaStream_t stream) {
  CUtensorMap mo;
  const bool acc_out = EPI == Epi::kAcc;
  const int esize = acc_out ? 4 : (int)sizeof(T);
  const CUtensorMapDataType odt = acc_out ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                          : (sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
  const CUtensorMapSwizzle oswz = esize == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tma_2d(&mo, p.g.out, odt, esize, (uint64_t)p.g.ldo, (uint64_t)p.g.M, kEpiChunk, 32, oswz))
    return cudaErrorInvalidValue;
  CUtensorMap mr = mo;   // unused unless there is a residual
  if (EPI == Epi::kStore && p.g.residual != nullptr &&
      !make_tma_2d(&mr, p.g.residual, odt, esize, (uint64_t)p.g.N, (uint64_t)p.g.M, kEpiChunk, 32, oswz))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(SmemLayout<(EPI == Epi::kAcc ? 4 : (int)sizeof(T)), UNP, RB>) + 1024;
  auto kern = tgemm_tc_kernel<EPI, T, UNP, RB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = std::min(tiles, num_sms());
  return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, stream, ma, mb[0], mb[1], mb[2], mo, mr, p);
}

}  // namespace

bool tgemm_tc_supported(const TGemmArgs& a, Epi epi) {
  if (epi != Epi::kStore && epi != Epi::kAcc && epi != Epi::kGlu) return false;
  if (a.K % 64 != 0 || a.N % HALF != 0) return false;   // 16-byte TMA row strides, whole 128-row halves
  if (epi == Epi::kGlu && a.nseg != 2) return false;
  if (a.residual != nullptr && a.nseg != 1) return false;
  return tma_available();
}

cudaError_t launch_tgemm_tc(const TGemmArgs& a, Epi epi, mmf_dtype dt, int* status, cudaStream_t stream) {
  if (a.M == 0) return cudaSuccess;
  if (!tgemm_tc_supported(a, epi)) return cudaErrorNotSupported;
  CUtensorMap ma, mb[3];
  if (!make_tma_2d(&ma, a.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.K, (uint64_t)a.M, BK, BM,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  bool unp = true;   // every segment has its one-byte copy
  for (int r = 0; r < a.nseg; ++r) unp = unp && a.wu[r] != nullptr;
  for (int r = 0; r < 3; ++r) {
    const int src = r < a.nseg ? r : 0;
    const bool ok = unp ? make_tma_2d(&mb[r], a.wu[src], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.K, (uint64_t)a.N,
                                      BK, HALF, CU_TENSOR_MAP_SWIZZLE_128B)
                        : make_tma_2d(&mb[r], a.w[src], CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)(a.K / 16),
                                      (uint64_t)a.N, BK / 16, HALF, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;
  }
  TcArgs p;
  p.g = a;
  p.status = status;
  p.wait_cycles = wait_limit_cycles();
  p.skip_it = (uint32_t)test_hook("MMF_TC_SKIP_KSTEP");
  p.m_tiles = ceil_div(a.M, BM);
  p.n_tiles = (epi == Epi::kGlu) ? ceil_div(a.N, HALF) : ceil_div(a.nseg * a.N, BN);
  const bool b = dt == MMF_BF16;
  // Short-K contractions with a residual (the o projection: K = 1024, 8
  // k-steps per tile) wait on the epilogue's residual loads: prefetch the whole
  // tile's residual (3-deep ring, 4 staging buffers per epilogue warp). 370M o
  // projection: 0.795 -> 0.744 ms per 24-layer step. Longer K (the down
  // projection) keeps the 4-deep ring, which its main loop needs more.
  if (epi == Epi::kStore && b && a.residual != nullptr && a.K <= 1024)
    return unp ? launch_typed<Epi::kStore, bf16, true, true>(ma, mb, p, stream)
               : launch_typed<Epi::kStore, bf16, false, true>(ma, mb, p, stream);
#define MMF_TC_LAUNCH(E)                                                                                      \
  (unp ? (b ? launch_typed<E, bf16, true>(ma, mb, p, stream) : launch_typed<E, float, true>(ma, mb, p, stream)) \
       : (b ? launch_typed<E, bf16, false>(ma, mb, p, stream) : launch_typed<E, float, false>(ma, mb, p, stream)))
  switch (epi) {
    case Epi::kStore: return MMF_TC_LAUNCH(Epi::kStore);
    case Epi::kAcc: return MMF_TC_LAUNCH(Epi::kAcc);
    case Epi::kGlu: return MMF_TC_LAUNCH(Epi::kGlu);
    default: return cudaErrorNotSupported;
  }
#undef MMF_TC_LAUNCH
}

}  // namespace mmf
