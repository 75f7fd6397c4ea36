// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/lmoe.h"

namespace lmoe {

// Every kernel of the library is launched with programmatic stream
// serialisation: the next kernel's blocks may be scheduled while this one
// finishes, and each kernel starts with griddepcontrol.wait (all of the
// preceding grid's work and memory visible) before any global access, so
// only the launch latency between kernels is hidden.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                            Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

void count_launch();                 // bump the library's kernel-launch counter
int device_sm_count();               // SMs of the current device (cached per device)

// One-time per-device setup of a kernel (function attributes persist per
// device): a bit per device ordinal below 64; devices from 64 on are set up
// on every call. Concurrent first calls may both run the (idempotent) setup.
inline bool device_configured(const std::atomic<uint64_t>& mask, int dev) {
  return dev >= 0 && dev < 64 && ((mask.load(std::memory_order_acquire) >> dev) & 1u);
}
inline void mark_configured(std::atomic<uint64_t>& mask, int dev) {
  if (dev >= 0 && dev < 64) mask.fetch_or(uint64_t(1) << dev, std::memory_order_release);
}

// ----- tensor-core GEMM (gemm_tc.cu) -----
struct TcOperand {
  const void* ptr;     // [groups][rows][k], k contiguous: BF16, or E4M3 bytes with elem == 1
  int64_t k;
  int64_t rows;
  int64_t groups;
  int elem = 2;        // bytes per element: 2 (BF16) or 1 (E4M3)
};

struct TcLaunch {
  int swap = 0;
  int grouped = 0;
  int rows = 0;                  // dense: activation rows
  int cols = 0;                  // output features
  int nseg = 1;
  TcOperand a[2] = {};
  TcOperand b[2] = {};
  int kblocks[2] = {0, 0};
  int a_kgroup[2] = {0, 0};
  int b_kgroup[2] = {0, 0};
  const int* offsets = nullptr;
  const int* padded_offsets = nullptr;
  int groups = 0;
  int64_t max_tiles = 0;         // host upper bound of the tile count (grid sizing)
  void* out = nullptr;
  int64_t ld_out = 0;
  const float* bias = nullptr;
  const float* row_scale = nullptr;
  const void* residual = nullptr;
  int64_t ld_res = 0;
  int epi = 0;
  int bn = 256;
  int ksplit = 1;                // >1: split-K with fp32 partials in `partial`, then a reduction
  float* partial = nullptr;      // [ksplit][rows][cols]
  int fp8 = 0;                   // 1: E4M3 operands (every segment), K blocks of 128
  const float* scale_a = nullptr;     // EPI_SQRELU_Q8 / EPI_SCALE: operand scales (device scalars)
  const float* scale_w = nullptr;
  const float* out_scale = nullptr;   // EPI_SQRELU_Q8: static scale of the E4M3 output
  // tc2_gemm only: a dense problem in the same launch, out_x = epi(x_act . x_wt^T)
  TcOperand x_act = {};          // [rows_x][k] activations
  TcOperand x_wt = {};           // [cols_x][k] weights, or [groups][cols_x][x_kgroup] with K split in groups
  int x_kgroup = 0;
  int rows_x = 0;
  int cols_x = 0;
  void* out_x = nullptr;
  int64_t ld_out_x = 0;
};

lmoe_status tc_gemm(const TcLaunch& L, uint32_t* err_word, cudaStream_t stream);
// Weight-major grouped GEMM on CTA pairs (M = 256 features per pair, up to 256
// tokens per tile); max_tiles bounds the pair-tile count.
lmoe_status tc2_gemm(const TcLaunch& L, uint32_t* err_word, cudaStream_t stream);

// ----- grouped NVFP4 expert GEMM (gemm_fp4.cu) -----
struct Fp4Launch {
  const void* a_codes = nullptr;     // [a_rows][k/2] packed E2M1 (padded expert-grouped rows)
  const uint8_t* a_sf = nullptr;     // MMA-tiled scales of A
  int64_t a_rows = 0;                // padded rows (multiple of 128)
  const void* b_codes = nullptr;     // [groups][cols][k/2]
  const uint8_t* b_sf = nullptr;     // per expert, MMA-tiled
  int64_t k = 0;
  int cols = 0;
  int groups = 0;
  const int* offsets = nullptr;
  const int* padded_offsets = nullptr;
  const float* in_scale = nullptr;   // device scalar, or [groups] with in_scale_grouped
  int in_scale_grouped = 0;
  const float* w_scale = nullptr;    // [groups]
  const float* out_scale = nullptr;  // device scalar (quant_out)
  const float* row_scale = nullptr;  // gates (GEMM 2)
  int quant_out = 0;                 // 1: relu^2 + NVFP4 codes/scales out; 0: BF16 out * gate
  int f32_out = 0;                   // with quant_out 0: fp32 out * gate instead of BF16
  // K-batched problems (BF16 out only): kgroups[2g], kgroups[2g+1] = first K
  // column (a multiple of 256) and 256-element K blocks of group g; A [a_rows][k]
  // and B [cols][k] are single matrices (k the total), group g's output
  // [a_rows][cols] at out + g * out_group_stride elements
  const int* kgroups = nullptr;
  int64_t out_group_stride = 0;
  void* out = nullptr;
  uint8_t* out_sf = nullptr;
  int64_t ld_out = 0;
};

lmoe_status fp4_gemm(const Fp4Launch& L, uint32_t* err_word, cudaStream_t stream);

// ----- fp32 SIMT GEMM (gemm_simt.cu) -----
struct SimtLaunch {
  int grouped = 0;
  int rows = 0;            // dense: activation rows; grouped: padded rows bound
  int cols = 0;
  int k = 0;
  const float* a = nullptr;       // [rows][lda]
  int64_t lda = 0;                // 0: k
  const float* b = nullptr;       // [groups][cols][k]
  const int* offsets = nullptr;
  const int* padded_offsets = nullptr;
  int groups = 1;
  float* out = nullptr;
  int64_t ld_out = 0;
  const float* bias = nullptr;
  const float* row_scale = nullptr;
  const float* residual = nullptr;
  int64_t ld_res = 0;
  int epi = 0;
  int accumulate = 0;      // 1: out += result (before the epilogue's rounding; fp32 so exact order)
};

lmoe_status simt_gemm(const SimtLaunch& L, uint32_t* err_word, cudaStream_t stream);

// ----- small kernels (lmoe_kernels.cu) -----
// x / w_router non-null: refine near-tied decisions with exact logits (see the
// kernel); refine_all: every candidate's logit exact (gates to fp32 rounding).
lmoe_status launch_topk(const float* logits, int64_t T, int N, int K, int32_t* idx, float* w, const void* x,
                        const void* w_router, const float* bias, int d, int act, uint32_t* err, cudaStream_t s,
                        int refine_all = 0);
// Slots per warp of the counting sort: the workspace path uses short chunks
// (more CTAs in flight); the fixed-scratch path keeps 1024 (fewer counters).
constexpr int kPermSlotsPerWarp = 128;
constexpr int kPermSlotsPerWarpStatic = 1024;
int permute_chunks(int64_t slots, int slots_per_warp = kPermSlotsPerWarp);
// scratch: (permute_chunks() + 1) * N int32. slot_row (optional, [T*K]): the
// padded row of each slot (-1 for a slot left out).
lmoe_status launch_permute(const int32_t* idx, int64_t T, int K, int N, int32_t* offsets,
                           int32_t* perm_src, int32_t* inv_perm, int32_t* padded_offsets,
                           int32_t* scratch, const float* topk_w, float* perm_gate,
                           uint32_t* err, cudaStream_t s, int slots_per_warp = kPermSlotsPerWarp,
                           int32_t* slot_row = nullptr);
lmoe_status launch_gather(const int32_t* idx, const int32_t* perm_src, const int32_t* offsets,
                          const int32_t* padded_offsets, int64_t slots, int K, const void* rows,
                          int64_t row_bytes, void* out_rows, const uint8_t* rows_sf,
                          uint8_t* out_sf, int N, cudaStream_t s);
lmoe_status launch_selftest_wait(uint32_t* err, long long limit_cycles, cudaStream_t s);
lmoe_status launch_combine(const void* y, int act, const int32_t* idx, const int32_t* inv_perm,
                           const int32_t* offsets, const int32_t* padded_offsets, const float* w,
                           const void* resid, void* c, int64_t T, int K, int N, int l, cudaStream_t s);
// BF16 rows -> NVFP4 (current amax) written at each row's K slot rows
// (slot_row [rows][K], -1 skips) with MMA-tiled scales; cols % 64 == 0, K <= 32.
lmoe_status launch_nvfp4_quantize_scatter(const void* in, int64_t rows, int cols, const int32_t* slot_row, int K,
                                          uint8_t* codes, uint8_t* sf, float* global_out, float* partials,
                                          int npartials, cudaStream_t s);
// Each of the n rows (row_bytes, a multiple of 16) copied to the padded rows
// of its K slots (slot_row[t*K+k]; -1 skips the slot).
lmoe_status launch_scatter_rows(const void* rows, int64_t n, int64_t row_bytes, const int32_t* slot_row, int K,
                                void* out, cudaStream_t s);
lmoe_status launch_nvfp4_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols,
                                  const float* global_in, uint8_t* codes, uint8_t* sf,
                                  float* global_out, int sf_layout, float* partials,
                                  int npartials, uint32_t* err, cudaStream_t s);
int nvfp4_partials(int64_t elems);
// Training-recipe NVFP4 quantiser (lmoe_train.cu): partials holds
// groups * nvfp4x_partials(out_rows * out_cols / 16) doubles. groups > 1:
// that many matrices of rows x cols, contiguous in `in`, codes and sf, each
// with its own global scale (global_out[g]); round to nearest only.
int nvfp4x_partials(int64_t blocks);
lmoe_status launch_nvfp4_quantize_ex(const void* in, int in_dtype, int64_t rows, int64_t cols, uint32_t flags,
                                     uint32_t rht_signs, uint64_t seed, uint32_t sr_stream, const float* global_in,
                                     uint8_t* codes, uint8_t* sf, float* global_out, int sf_layout, double* partials,
                                     cudaStream_t s, int64_t out_pitch = 0, int groups = 1);
// Codes and MMA-tiled scales of `groups` [rows][cols] matrices quantised with
// 16 x 16 blocks -> those of their transposes (rows, cols multiples of 128).
lmoe_status launch_nvfp4_transpose2d(const uint8_t* codes, const uint8_t* sf, int64_t groups, int64_t rows,
                                     int64_t cols, uint8_t* codes_t, uint8_t* sf_t, cudaStream_t s);
// Ragged groups: group g quantises input rows [gtab[6g], gtab[6g] + gtab[6g+1])
// of a [*][cols] input as one matrix (own global scale global_out[g], SR
// stream stream0 + g * stream_step), codes at codes + gtab[6g+2], scales at
// sf + gtab[6g+3], output pitch gtab[6g+4] (0: the output's columns);
// gtab[6g+5] (the rows holding data) is informational.
// ld > 0 (a multiple of 64): every group writes into one matrix of ld-element
// rows (codes at ld / 2 bytes per row, MMA-tiled atoms over ld / 64 column
// groups), its offsets naming its first column. rows_max / pitch_max bound
// every group's rows and pitch (grid sizing); partials holds
// groups * nvfp4x_partials(out_rows_max * pitch_max / 16) doubles.
lmoe_status launch_nvfp4_quantize_groups(const void* in, int in_dtype, int64_t rows_max, int64_t cols,
                                         uint32_t flags, uint32_t rht_signs, uint64_t seed, uint32_t stream0,
                                         uint32_t stream_step, const int64_t* gtab, int groups, int64_t pitch_max,
                                         int64_t ld, uint8_t* codes, uint8_t* sf, float* global_out, int sf_layout,
                                         double* partials, cudaStream_t s);
// Dense BF16 GEMM on the tensor cores (lmoe_api.cu): out[rows][cols] =
// epi(x[rows][k] . w[cols][k]^T), token-major tiles, or weight-major ones for
// rows <= 64 (split-K into `partial` when given). epi: EPI_* of gemm_tc.cuh
// (EPI_F32_BIAS: fp32 out (+ bias); EPI_BF16; EPI_ADD_RES: + residual, BF16).
lmoe_status dense_bf16(const void* x, int64_t rows, const void* w, int cols, int64_t k, void* out,
                       int64_t ld_out, int epi, const float* bias, const void* residual, int64_t ld_res,
                       float* partial, uint32_t* err, cudaStream_t s);
// Routed experts' backward under the NVFP4 training recipe (lmoe_train_experts.cu):
// the body of lmoe_expert_backward_nvfp4 without its argument checks; ws holds
// at least expert_backward_ws(cfg, counts) bytes (first 256 the error word);
// o_out (nullable): receives the recomputed expert outputs o, fp32 [P][l];
// err_word (nullable): the error word to report into instead of ws's own.
size_t expert_backward_ws(const lmoe_config* cfg, const int32_t* counts);
size_t expert_backward_ws_bound(const lmoe_config* cfg);   // any routing of cfg->T tokens
lmoe_status expert_backward_core(const lmoe_config* cfg, const int32_t* counts, const int32_t* offsets,
                                 const int32_t* padded_offsets, const uint8_t* z_codes, const uint8_t* z_sf,
                                 const float* z_global, const void* w1, const void* w2, const float* a_global,
                                 const float* gate, const float* dy, uint64_t seed, uint32_t rht_signs, void* dz,
                                 float* dgate, void* dw1, void* dw2, void* ws, float* o_out, uint32_t* err_word,
                                 cudaStream_t s, const float* dy_tok = nullptr, const int32_t* perm_src = nullptr,
                                 int K = 0);
// FP8 E4M3 codes of in / s with one FP32 scale per tensor (scale_in, or the
// tensor's amax / 448 when scale_in is null; scale_out receives it).
lmoe_status launch_fp8_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols, const float* scale_in,
                                uint8_t* codes, float* scale_out, float* partials, int npartials, cudaStream_t s);

}  // namespace lmoe
