// Internal launchers of the mmf CUDA library. Not part of the C ABI.
#pragma once

#include <cuda.h>

#include <algorithm>
#include <utility>

#include "common.cuh"

namespace mmf {

constexpr int kQuantPartials = 592;   // CTAs of the absmean partial-sum pass (4 x 148 SMs)

// TMA tensor maps (host): a 2-D row-major [rows, cols] array of esize-byte elements.
bool tma_available();
bool make_tma_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols,
                 uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);
int num_sms();

// Launch `kern` with programmatic stream serialization (the kernel must call
// pdl_wait() before touching anything a predecessor wrote or reads).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Message returned by mmf_last_error() on this host thread.
void set_last_error(const char* msg);

size_t quantize_weights_ws_bytes();
// Packed codes [N, K/16] -> one byte per weight [N, K] holding the stored code
// w + 1 (K % 16 == 0; `out` 16-byte aligned).
cudaError_t launch_unpack_codes(const uint32_t* packed, int N, int K, uint8_t* out, cudaStream_t stream);
cudaError_t launch_quantize_weights(const float* W, int N, int K, uint32_t* packed, float* gamma, void* ws,
                                    cudaStream_t stream);

// `status` (nullable) is the device status word for bounded-wait timeouts.
// Optionally, as side work for a later kernel, it sets `fill_bytes` bytes at
// `fill` (16-byte aligned) to 0xff, stream-ordered like a memset.
cudaError_t launch_rmsnorm_quant(const void* x, mmf_dtype dt, int M, int K, const float* gain, float eps,
                                 int8_t* q, float* scale, int32_t* qsum, int* status, cudaStream_t stream,
                                 void* fill = nullptr, size_t fill_bytes = 0);

// Epilogues of the ternary contraction.
enum class Epi : int {
  kStore = 0,     // y[m, seg*N + n] = acc*gamma_seg/s + bias (+ residual[m, n] when 1 segment)
  kAcc = 1,       // int32 acc[m, n]
  kScanStep = 2,  // 3 segments f,c,g: one MLGRU step, h[m, n] in place, o'[m, n]
  kGlu = 3,       // 2 segments gate,up: p[m, n] = SiLU(u) * v
};

struct TGemmArgs {
  const uint32_t* w[3];     // packed ternary weights per segment, [N, K/16]
  const uint8_t* wu[3];     // optional: the same codes one byte per weight, [N, K] (tcgen05 path reads
                            // them with TMA instead of unpacking the packed words); null = not available
  const float* gamma[3];    // per-segment scale (device scalar)
  const float* bias[3];     // per-segment bias [N] or null
  int nseg;                 // 1..3
  int N;                    // rows per segment
  int K;
  const int8_t* q;          // [M, K] activation codes
  const float* s;           // [M] activation scales
  const int32_t* qsum;      // [M] row sums of q
  int M;
  void* out;                // see Epi
  int ldo;                  // leading dimension of out (elements)
  const void* residual;     // [M, N] in the activation dtype, or null
  float* h;                 // kScanStep: [M, N] fp32 state, updated in place
  // Decode contraction only: when x is set, the kernel quantises the token
  // rows x [M, K] (activation dtype, RMSNorm gain `gain` or null, `eps`)
  // itself and q/s/qsum above are not read; q_out/s_out/qsum_out (nullable)
  // then receive the codes, scales and sums.
  const void* x;
  const float* gain;
  float eps;
  int8_t* q_out;
  float* s_out;
  int32_t* qsum_out;
};



// mma.sync-based contraction (weights as the 16-row A operand, tokens as N=8 tiles).
cudaError_t launch_tgemm_mma(const TGemmArgs& a, Epi epi, mmf_dtype dt, cudaStream_t stream);
// Whether launch_tgemm_mma can quantise the token rows itself (TGemmArgs::x):
// up to 16 tokens whose rows (esize bytes per element) and codes fit the
// kernel's shared memory.
bool tgemm_mma_fused_quant_supported(int M, int K, int esize);

// tcgen05 (TMEM) contraction for prefill-sized token counts. Needs K % 64 == 0
// and N % 128 == 0; `status` is the device status word for bounded-wait timeouts.
bool tgemm_tc_supported(const TGemmArgs& a, Epi epi);
cudaError_t launch_tgemm_tc(const TGemmArgs& a, Epi epi, mmf_dtype dt, int* status, cudaStream_t stream);

// The same contraction on SM pairs (tcgen05 cta_group::2, 256-token tiles); needs M >= 256.
bool tgemm_tc2_supported(const TGemmArgs& a, Epi epi);
cudaError_t launch_tgemm_tc2(const TGemmArgs& a, Epi epi, mmf_dtype dt, int* status, cudaStream_t stream);

// Prefill token mixer in one kernel: the f|c|g contraction (a.nseg == 3, rows
// of the three matrices for the same channels) with the MLGRU gates and
// recurrence in its epilogue; writes o' [M, d] (a.out, activation dtype) and
// updates the state h [B, d]. Needs T % 128 == 0 and d % 64 == 0. `ws` holds
// tgemm_tc_mlgru_ws_bytes(B, T, d) bytes that reset_tgemm_tc_mlgru_ws() must
// prepare (stream-ordered) before every launch.
bool tgemm_tc_mlgru_supported(const TGemmArgs& a, int T, int d);
size_t tgemm_tc_mlgru_ws_bytes(int B, int T, int d);
cudaError_t reset_tgemm_tc_mlgru_ws(void* ws, int B, int T, int d, cudaStream_t stream);
cudaError_t launch_tgemm_tc_mlgru(const TGemmArgs& a, mmf_dtype dt, int T, int d, float* h, void* ws, int* status,
                                  cudaStream_t stream);

// One decode step (T = 1, M <= 8 tokens) of a whole block in one cooperative
// launch (grid = one CTA per SM): stage 0 quantises x with st[0].gain and runs
// f|c|g (3 segments, N = d) with the MLGRU step (h in place, o' -> og); stage 1
// quantises og and runs o (+ x) -> y1; stage 2 quantises y1 and runs gate|up
// (2 segments, N = I) with SiLU(gate) * up -> p; stage 3 quantises p and runs
// down (+ y1) -> y. `bar` holds 256 bytes (words 0 and 32 used) that are zero
// between launches.
constexpr int kDecodeMaxTiles = 4;   // 16-row weight tiles per CTA and stage
struct DecodeStage {
  const uint32_t* w[3];     // packed codes per segment, [N, K/16]
  const float* gamma[3];    // per-segment scale (device scalar)
  const float* bias[3];     // per-segment bias [N] or null
  const float* gain;        // RMSNorm gain [K] of the stage's input, or null
  int nseg, N, K;
};
struct DecodeBlockArgs {
  DecodeStage st[4];        // f|c|g, o, gate|up, down
  const void* x;            // [M, d] block input (activation dtype)
  void* og;                 // [M, d] o'
  void* y1;                 // [M, d] token-mixer output
  void* p;                  // [M, I] GLU product
  void* y;                  // [M, d] block output
  float* h;                 // [M, d] recurrent state
  int M, d, I;
  float eps;
  unsigned* bar;            // grid-barrier words (counter, generation)
  int* status;              // device status word (code 4: a barrier wait gave up)
  int slot_bytes;           // set by the launcher
};
bool decode_block_supported(const DecodeBlockArgs& a, mmf_dtype dt);
cudaError_t launch_decode_block(DecodeBlockArgs a, mmf_dtype dt, cudaStream_t stream);

// Chunk-parallel MLGRU scan; `ws` holds mlgru_scan_ws_bytes(B, T, d) bytes of
// scratch, which reset_mlgru_scan_ws() must prepare (stream-ordered) before
// every launch; launch_mlgru_scan() itself enqueues only the kernel (launched
// as a programmatic dependent of the kernel before it). `status` is the device
// status word for bounded-wait timeouts.
size_t mlgru_scan_ws_bytes(int B, int T, int d);
cudaError_t reset_mlgru_scan_ws(void* ws, int B, int T, int d, cudaStream_t stream);
cudaError_t launch_mlgru_scan(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, void* o, void* ws,
                              int* status, cudaStream_t stream);

}  // namespace mmf
