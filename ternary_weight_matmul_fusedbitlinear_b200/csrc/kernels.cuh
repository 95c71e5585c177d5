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
// Bound of the kernels' device-side waits, in SM cycles: about 1 s at 2 GHz, or
// MMF_WAIT_LIMIT_US microseconds when set (tests make waits run out quickly).
long long wait_limit_cycles();
// Integer test hook from the environment variable `name` (-1 when unset).
int test_hook(const char* name);

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
  void* pre_out;            // kScanStep, nullable: the stored f~, c~, g~ values, [M, 3, N] (activation dtype)
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

// One decode step (T = 1) of L consecutive blocks in one cooperative launch
// (decode_step.cu). Per-block device descriptor, built at block creation:
struct DecodeLayerDesc {
  const uint32_t* w[7];     // packed codes: f, c, g, o, gate, up, down
  const float* gamma[7];    // their scales (device scalars)
  const float* bias[7];     // their biases, or null
  const float* gain[4];     // RMSNorm gains of the four quantised inputs (x, o', y1, p), or null
};
constexpr int kDecodeMaxLayers = 32;   // layers per launch
constexpr int kDecodeTiles = 3;        // 16-row tiles per CTA and stage
constexpr int kDecodeMaxSlots = 4;     // weight ring depth
struct DecodeStepArgs {
  const DecodeLayerDesc* layer[kDecodeMaxLayers];
  const void* x;            // [M, d] input of the first layer (activation dtype)
  void* y;                  // [M, d] output of the last layer
  float* h;                 // state [L_state, M, d]; this launch uses layers layer0 .. layer0 + L - 1
  uint8_t* xbuf;            // exchange buffers: per state layer decode_xlayer_bytes(M, d, I) bytes
  unsigned* parity;         // per state layer: which buffer set the next launch writes
  int* abort_word;          // raised by a CTA that gave up a wait; zero between launches
  int* status;              // device status word (codes 5, 6)
  mmf_block_debug dbg;      // L == 1 only: optional copies of the intermediates
  size_t xlayer_bytes, xset_bytes;
  long long wait_cycles;    // bound of every wait, in SM clock cycles
  float eps;
  int L, layer0, M, d, I;
  int xI;                   // inner size the exchange buffers were allocated for (>= I)
  int nslot, slot_bytes, qpitch, desc_bytes, codes_bytes;   // set by the launcher
  int skip_cta;             // test hook: this CTA never publishes its first stage (-1: none)
};
// Bytes of exchange buffers (both sets) per state layer.
size_t decode_xlayer_bytes(int M, int d, int I);
bool decode_step_supported(int M, int d, int I, int L, mmf_dtype dt);
// Grid of the launch: one CTA per SM, at most one per 16-row tile of the widest stage.
int decode_step_grid(int d, int I);
cudaError_t launch_decode_step(DecodeStepArgs a, mmf_dtype dt, cudaStream_t stream);

// MLGRU gates + scan; one CTA per (sequence, 64 or 32 channels) walks the
// sequence's chunks in order. Launched as a programmatic dependent of the
// kernel before it. `status` is the device status word for bounded-wait
// timeouts. mlgru_scan_ws_bytes() is the scratch the C ABI's workspace size
// reports (the kernel uses none).
size_t mlgru_scan_ws_bytes(int B, int T, int d);
cudaError_t launch_mlgru_scan(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, void* o, int* status,
                              cudaStream_t stream);
// The same recurrence with the g_norm output gate: the scan writes
// v = swish(g~) h (fp32) and per-(token, channel block) sums of h^2 into `ws`
// (mlgru_scan_gnorm_ws_bytes), then a row kernel writes
// o' = v / sqrt(mean h^2 + eps) * gain in dtype. Two launches, each a
// programmatic dependent of the one before.
size_t mlgru_scan_gnorm_ws_bytes(int B, int T, int d);
cudaError_t launch_mlgru_scan_gnorm(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, const float* gain,
                                    float eps, void* o, void* ws, int* status, cudaStream_t stream);
// Backward of the scan (training): the forward states h_t (fp32, into `ws`,
// mlgru_scan_bwd_ws_bytes), then a reverse chunked scan writing dL/d(f~, c~, g~)
// [B, T, 3, d] in dtype and dL/dh0 [B, d] (also the forward's carried-state
// scratch until the reverse scan overwrites it).
size_t mlgru_scan_bwd_ws_bytes(int B, int T, int d);
cudaError_t launch_mlgru_scan_bwd(const void* pre, mmf_dtype dt, int B, int T, int d, const float* h0,
                                  const void* dout, const float* dhT, const float* hs, void* dpre, float* dh0,
                                  void* ws, int* status, cudaStream_t stream);
// The forward scan (sigmoid gate) that also stores the states h_t in fp32 into
// hs [B, T, d] for a later backward; o (o') may be null.
cudaError_t launch_mlgru_scan_states(const void* pre, mmf_dtype dt, int B, int T, int d, float* h, void* o, float* hs,
                                     int* status, cudaStream_t stream);
// Inside a block: the same scan, then one row kernel that forms o' and
// quantises it for the o projection (RMSNorm gain qgain, eps) into q / scale /
// qsum with the standalone quantiser's row routine; o' is written only when
// `o` is not null.
cudaError_t launch_mlgru_scan_gnorm_quant(const void* pre, mmf_dtype dt, int B, int T, int d, float* h,
                                          const float* gain, float eps_g, void* o, void* ws, int* status,
                                          const float* qgain, float eps, int8_t* q, float* scale, int32_t* qsum,
                                          cudaStream_t stream);

// Model ends: token embedding lookup (one warp per row; an id outside [0, V)
// writes zeros and records status code 8) and the greedy next token (one CTA
// per logit row, lowest index on ties). Both are programmatic dependents.
cudaError_t launch_embed(const int32_t* ids, int M, const void* table, int V, int d, mmf_dtype dt, void* x,
                         int* status, cudaStream_t stream);
cudaError_t launch_argmax(const void* logits, mmf_dtype dt, int M, int V, int32_t* ids, cudaStream_t stream);

}  // namespace mmf
