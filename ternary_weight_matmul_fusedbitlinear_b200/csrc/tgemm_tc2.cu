// Prefill ternary contraction on an SM pair: tcgen05 kind::i8 with
// cta_group::2 (one 256-token x 256-column tile per CTA pair).
//
// Same arithmetic as the single-SM kernel (tgemm_tc.cu): "MatMul-free
// language models" (DataCamp blog), section "Replacing MatMul with ternary
// operations" — with weights in {-1,0,1} the contraction is exact integer
// work; the stored code w+1 is multiplied as an unsigned byte and the token's
// code sum is subtracted in the epilogue.
//
// Why a pair: each CTA holds half of the activation tile (its 128 tokens) and
// half of the weight tile (128 of the 256 output columns), so every SM unpacks
// and stores only half as many weight bytes per multiply-accumulate as on one
// SM, and the single MMA instruction (M = 256) covers both halves.
//
// Roles per CTA (448 threads), as in the single-SM kernel:
//   warp 0      TMA: this CTA's activation half (cta_group::2 copy signalling
//               the leader's barrier) and its 128 packed weight rows
//   warp 1      TMEM allocation (both CTAs); in the leader (rank 0) also the
//               single MMA-issuing thread
//   warps 2..9  epilogue of this CTA's 128 accumulator rows
//   warps 10-13 unpack of this CTA's 128 weight rows
// Barriers that collect both CTAs (activation halves landed, both halves
// unpacked, both epilogues done) live in the leader; the MMA commits arrive in
// both CTAs through the cluster multicast form of tcgen05.commit. No TMA load
// uses cluster multicast. Every wait is bounded.
#include "kernels.cuh"
#include "umma.cuh"

namespace mmf {

namespace {

constexpr int BMH = 128;                 // tokens per CTA (256 per pair)
constexpr int BN = 256, BK = 128;
constexpr int HALF = BN / 2;             // weight rows per CTA
constexpr int A_BYTES = BMH * BK;        // 16 KiB
constexpr int BP_BYTES = HALF * BK / 4;  // 4 KiB
constexpr int BU_BYTES = HALF * BK;      // 16 KiB
constexpr int NB = 3;
constexpr int kEpiWarps = 8, kEpiWarp0 = 2, kUnpackWarp0 = 10, kUnpackWarps = 4;
constexpr int kThreads = (kUnpackWarp0 + kUnpackWarps) * 32;
constexpr int kEpiChunk = 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc2 = umma_idesc_i8(2 * BMH, BN);

template <int OB>
struct __align__(1024) Smem2 {
  static constexpr int NS = OB == 2 ? 6 : 4;
  static constexpr int kStageBytes = 32 * kEpiChunk * OB;
  uint8_t a[NS][A_BYTES];
  uint8_t bu[NB][BU_BYTES];
  uint8_t stage[kEpiWarps][2][kStageBytes];
  uint32_t bp[NS][BP_BYTES / 4];
  uint64_t a_full[NS];      // leader: both activation halves of stage s landed
  uint64_t bp_full[NS];     // this CTA's packed codes of stage s landed
  uint64_t tma_empty[NS];   // stage s free again (MMA commit, both CTAs)
  uint64_t bu_full[NB];     // leader: both CTAs unpacked slot u (one arrival per unpack warp)
  uint64_t bu_empty[NB];    // slot u free again (MMA commit, both CTAs)
  uint64_t tmem_full[2];    // accumulator ready (MMA commit, both CTAs)
  uint64_t tmem_empty[2];   // leader: both CTAs' epilogues read it (one arrival per epilogue warp)
  uint64_t res_full[kEpiWarps];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort_flag;
};

// ---------------------------------------------------------------- cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address, in the cluster window, of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t caddr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait with cluster-scope acquire (arrivals may come from the peer CTA).
static __device__ __noinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                 int* status) {
  if (mbar_try_wait_cl(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort_flag = 1;
      if (status) atomicExch(status, 1);
      return false;
    }
  }
}
// TMA load into this CTA's shared memory whose completion is counted on the
// leader's barrier `leader_bar` (a cluster-window address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int x, int y,
                                                 uint32_t leader_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(leader_bar)
      : "memory");
}
__device__ __forceinline__ void umma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kIdesc2), "r"(accum)
      : "memory");
}
// Arrive on the barrier at this offset in both CTAs once the issued MMAs complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}

struct Tc2Args {
  TGemmArgs g;
  int m_tiles, n_tiles;   // m_tiles counts 256-token pair tiles
  int* status;
};

// Weight rows feeding this CTA's half `h` (= its cluster rank) of tile nt.
__device__ __forceinline__ void half_source2(const Tc2Args& p, Epi epi, int nt, int h, int& seg, int& row0) {
  if (epi == Epi::kGlu) {
    seg = h;
    row0 = nt * HALF;
  } else {
    const int gcol = nt * BN + h * HALF;
    const int total = p.g.nseg * p.g.N;
    if (gcol >= total) {
      seg = p.g.nseg - 1;
      row0 = p.g.N;
    } else {
      seg = gcol / p.g.N;
      row0 = gcol % p.g.N;
    }
  }
}

template <Epi EPI, typename T>
__global__ void __launch_bounds__(kThreads, 1)
    tgemm_tc2_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b0,
                     const __grid_constant__ CUtensorMap map_b1, const __grid_constant__ CUtensorMap map_b2,
                     const __grid_constant__ CUtensorMap map_out, const __grid_constant__ CUtensorMap map_res,
                     const Tc2Args p) {
  constexpr int OB = EPI == Epi::kAcc ? 4 : (int)sizeof(T);
  using Smem = Smem2<OB>;
  constexpr int NS = Smem::NS;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  volatile int* abort_flag = &sm.abort_flag;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int n_tiles_total = p.m_tiles * p.n_tiles;
  const int nk = ceil_div(p.g.K, BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.a_full[s], 1);
      mbar_init(&sm.bp_full[s], 1);
      mbar_init(&sm.tma_empty[s], 1);
    }
    for (int u = 0; u < NB; ++u) {
      mbar_init(&sm.bu_full[u], 2 * kUnpackWarps);
      mbar_init(&sm.bu_empty[u], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.tmem_full[a], 1);
      mbar_init(&sm.tmem_empty[a], 2 * kEpiWarps);
    }
    for (int w = 0; w < kEpiWarps; ++w) mbar_init(&sm.res_full[w], 1);
    mbar_init(&sm.mma_drain, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&map_a);
    prefetch_tmap(&map_out);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const CUtensorMap* maps[3] = {&map_b0, &map_b1, &map_b2};
      uint32_t it = 0;
      bool ok = true;
      for (int tile = pair; tile < n_tiles_total && ok; tile += npairs) {
        const int mt = tile / p.n_tiles, nt = tile % p.n_tiles;
        int seg, row0;
        half_source2(p, EPI, nt, (int)rank, seg, row0);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % NS;
          if (!mbar_wait_cl(&sm.tma_empty[s], ((it / NS) & 1) ^ 1, abort_flag, p.status)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&sm.a_full[s], 2 * A_BYTES);
          tma_load_2d_pair(sm.a[s], &map_a, kb * BK, mt * 2 * BMH + (int)rank * BMH, cluster_addr(&sm.a_full[s], 0));
          mbar_arrive_expect_tx(&sm.bp_full[s], BP_BYTES);
          tma_load_2d(sm.bp[s], maps[seg], kb * (BK / 16), row0, &sm.bp_full[s]);
        }
      }
      // this CTA's packed-code copies land before exit (activation halves are
      // drained by the leader's MMA thread, which waits for them)
      for (uint32_t j = (it > NS ? it - NS : 0); j < it; ++j)
        mbar_wait_cl(&sm.bp_full[j % NS], (j / NS) & 1, abort_flag, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (leader && lane == 0) {
      uint32_t it = 0, tl = 0;
      bool ok = true;
      for (int tile = pair; tile < n_tiles_total && ok; tile += npairs, ++tl) {
        const int acc = tl & 1;
        const uint32_t acc_ph = (tl >> 1) & 1;
        if (!mbar_wait_cl(&sm.tmem_empty[acc], acc_ph ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % NS, u = it % NB;
          if (!mbar_wait_cl(&sm.bu_full[u], (it / NB) & 1, abort_flag, p.status) ||
              !mbar_wait_cl(&sm.a_full[s], (it / NS) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = umma_desc_sw128(smem_u32(sm.a[s]));
          const uint64_t bdesc = umma_desc_sw128(smem_u32(sm.bu[u]));
#pragma unroll
          for (int j = 0; j < BK / 32; ++j)
            umma_i8_pair(d_tmem, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), (kb | j) != 0);
          umma_commit_pair(&sm.tma_empty[s]);
          umma_commit_pair(&sm.bu_empty[u]);
        }
        if (ok) umma_commit_pair(&sm.tmem_full[acc]);
      }
      umma_commit_pair(&sm.mma_drain);
      mbar_wait_cl(&sm.mma_drain, 0, abort_flag, nullptr);
    }
  } else if (warp >= kUnpackWarp0) {
    // ------------------------------------------------------------ unpack this CTA's 128 weight rows
    const int tid = threadIdx.x - kUnpackWarp0 * 32;   // 0..127
    const uint32_t leader_bu_full0 = cluster_addr(&sm.bu_full[0], 0);
    uint32_t it = 0;
    bool ok = true;
    for (int tile = pair; tile < n_tiles_total && ok; tile += npairs) {
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % NS, u = it % NB;
        if (!mbar_wait_cl(&sm.bp_full[s], (it / NS) & 1, abort_flag, p.status) ||
            !mbar_wait_cl(&sm.bu_empty[u], ((it / NB) & 1) ^ 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        const uint4* src = reinterpret_cast<const uint4*>(sm.bp[s]);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int id = tid + kUnpackWarps * 32 * i;      // 256 (row, half-row) units
          const int n = id >> 1, h = id & 1;
          const uint4 w4 = src[id];
          const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
          uint8_t* dst = sm.bu[u] + n * BK;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * h + e;
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
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(leader_bu_full0 + (uint32_t)(u * sizeof(uint64_t)));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (8 warps) of this CTA's rows
    const int ew = warp - kEpiWarp0;
    const int quarter = warp & 3;
    const int group = ew >> 2;
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t leader_tmem_empty0 = cluster_addr(&sm.tmem_empty[0], 0);
    uint8_t* stage0 = sm.stage[ew][0];
    uint8_t* stage1 = sm.stage[ew][1];
    int nst = 0;
    uint32_t nres = 0;
    uint32_t tl = 0;
    const bool has_res = EPI == Epi::kStore && p.g.residual != nullptr;
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
    for (int tile = pair; tile < n_tiles_total && alive; tile += npairs, ++tl) {
      const int mt = tile / p.n_tiles, nt = tile % p.n_tiles;
      const int acc = tl & 1;
      const uint32_t acc_ph = (tl >> 1) & 1;
      const bool got = mbar_wait_cl(&sm.tmem_full[acc], acc_ph, abort_flag, p.status);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int mbase = mt * 2 * BMH + (int)rank * BMH;
      const int m = mbase + row_in_tile;
      const int y0 = mbase + quarter * 32;
      const bool row_ok = m < p.g.M;
      const float inv_s = row_ok ? 1.0f / p.g.s[m] : 0.0f;
      const int qs = row_ok ? p.g.qsum[m] : 0;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      if constexpr (EPI == Epi::kGlu) {
        const float sc_u = *p.g.gamma[0] * inv_s, sc_v = *p.g.gamma[1] * inv_s;
        for (int cc = 0; cc < 2; ++cc) {
          const int c = group * 2 + cc;
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
        const int h = group;
        int seg, row0;
        half_source2(p, EPI, nt, h, seg, row0);
        if (nt * BN + h * HALF < p.g.nseg * p.g.N) {
          const float sc = *p.g.gamma[seg] * inv_s;
          const float* bias = p.g.bias[seg];
          for (int c = 0; c < HALF / kEpiChunk; ++c) {
            const int n0 = row0 + 32 * c;
            const int x0 = seg * p.g.N + n0;
            uint8_t* buf;
            claim(buf);
            if (has_res && lane == 0) {
              mbar_arrive_expect_tx(&sm.res_full[ew], 32 * kEpiChunk * OB);
              tma_load_2d(buf, &map_res, n0, y0, &sm.res_full[ew]);
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
                const bool ok = mbar_wait(&sm.res_full[ew], nres & 1, abort_flag, p.status);
                ++nres;
                if (!__all_sync(0xffffffffu, ok)) { alive = false; break; }
                add_staged_row(buf, lane, out, (T*)nullptr);
                __syncwarp();
              }
              stage_row(buf, lane, out, (T*)nullptr);
            }
            release(x0, y0, buf);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(leader_tmem_empty0 + (uint32_t)(acc * sizeof(uint64_t)));
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // the leader's MMAs (which read this CTA's smem) and all remote arrivals are done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

template <Epi EPI, typename T>
cudaError_t launch_pair(const CUtensorMap& ma, const CUtensorMap (&mb)[3], const Tc2Args& p, cudaStream_t stream) {
  constexpr bool acc_out = EPI == Epi::kAcc;
  constexpr int esize = acc_out ? 4 : (int)sizeof(T);
  CUtensorMap mo;
  const CUtensorMapDataType odt = acc_out ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                          : (sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
  const CUtensorMapSwizzle oswz = esize == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tma_2d(&mo, p.g.out, odt, esize, (uint64_t)p.g.ldo, (uint64_t)p.g.M, kEpiChunk, 32, oswz))
    return cudaErrorInvalidValue;
  CUtensorMap mr = mo;
  if (EPI == Epi::kStore && p.g.residual != nullptr &&
      !make_tma_2d(&mr, p.g.residual, odt, esize, (uint64_t)p.g.N, (uint64_t)p.g.M, kEpiChunk, 32, oswz))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem2<esize>) + 1024;
  auto kern = tgemm_tc2_kernel<EPI, T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_clusters = 0;
  cfg.gridDim = dim3(2);
  if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess || max_clusters < 1)
    max_clusters = num_sms() / 2;
  const int tiles = p.m_tiles * p.n_tiles;
  const int pairs = std::max(1, std::min(tiles, max_clusters));
  cfg.gridDim = dim3(2 * pairs);
  return cudaLaunchKernelEx(&cfg, kern, ma, mb[0], mb[1], mb[2], mo, mr, p);
}

}  // namespace

bool tgemm_tc2_supported(const TGemmArgs& a, Epi epi) { return a.M >= 2 * BMH && tgemm_tc_supported(a, epi); }

cudaError_t launch_tgemm_tc2(const TGemmArgs& a, Epi epi, mmf_dtype dt, int* status, cudaStream_t stream) {
  if (a.M == 0) return cudaSuccess;
  if (!tgemm_tc2_supported(a, epi)) return cudaErrorNotSupported;
  CUtensorMap ma, mb[3];
  if (!make_tma_2d(&ma, a.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.K, (uint64_t)a.M, BK, BMH,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  for (int r = 0; r < 3; ++r) {
    const int src = r < a.nseg ? r : 0;
    if (!make_tma_2d(&mb[r], a.w[src], CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)(a.K / 16), (uint64_t)a.N, BK / 16,
                     HALF, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  Tc2Args p;
  p.g = a;
  p.status = status;
  p.m_tiles = ceil_div(a.M, 2 * BMH);
  p.n_tiles = (epi == Epi::kGlu) ? ceil_div(a.N, HALF) : ceil_div(a.nseg * a.N, BN);
  const bool b = dt == MMF_BF16;
  switch (epi) {
    case Epi::kStore:
      return b ? launch_pair<Epi::kStore, bf16>(ma, mb, p, stream) : launch_pair<Epi::kStore, float>(ma, mb, p, stream);
    case Epi::kAcc:
      return b ? launch_pair<Epi::kAcc, bf16>(ma, mb, p, stream) : launch_pair<Epi::kAcc, float>(ma, mb, p, stream);
    case Epi::kGlu:
      return b ? launch_pair<Epi::kGlu, bf16>(ma, mb, p, stream) : launch_pair<Epi::kGlu, float>(ma, mb, p, stream);
    default:
      return cudaErrorNotSupported;
  }
}

}  // namespace mmf
