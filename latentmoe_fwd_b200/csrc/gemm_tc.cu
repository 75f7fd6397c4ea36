// Host side of the tcgen05 GEMM: TMA tensor maps, tile-size and epilogue
// dispatch, persistent-grid sizing.
#include <mutex>

#include "gemm_tc.cuh"
#include "gemm_tc2.cuh"
#include "lmoe_internal.h"

namespace lmoe {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D map over a tensor [groups][rows][k] (k contiguous) of BF16 (box = 64 x
// box_rows x 1) or E4M3 bytes (box = 128 x box_rows x 1): 128 bytes of K per
// row either way, 128-byte swizzle, zero fill out of bounds.
static bool make_map_bf16(CUtensorMap* map, const TcOperand& op, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || !op.ptr || (op.elem != 1 && op.elem != 2)) return false;
  const int64_t eb = op.elem;
  if ((reinterpret_cast<uintptr_t>(op.ptr) & 15) != 0 || (op.k * eb) % 16 != 0) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(op.k), static_cast<cuuint64_t>(op.rows),
                        static_cast<cuuint64_t>(op.groups)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(op.k * eb), static_cast<cuuint64_t>(op.rows * op.k * eb)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, eb == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                   const_cast<void*>(op.ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int STAGES, int EPI>
static lmoe_status launch_tc(const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1,
                             const CUtensorMap& b1, const CUtensorMap& bs, const TcParams& p, int grid,
                             cudaStream_t s) {
  using Sm = TcSmem<BN, STAGES>;
  auto kern = tc_gemm_kernel<BN, STAGES, EPI>;
  constexpr int smem = Sm::kBytes;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!device_configured(configured, dev)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return LMOE_ERR_CUDA;
    mark_configured(configured, dev);
  }
  launch_k(kern, dim3(grid), dim3(192), smem, s, a0, b0, a1, b1, bs, p);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

template <int BN, int STAGES>
static lmoe_status dispatch_epi(int epi, const CUtensorMap* m, const TcParams& p, int grid, cudaStream_t s) {
  switch (epi) {
    case EPI_F32_BIAS: return launch_tc<BN, STAGES, EPI_F32_BIAS>(m[0], m[1], m[2], m[3], m[4], p, grid, s);
    case EPI_BF16: return launch_tc<BN, STAGES, EPI_BF16>(m[0], m[1], m[2], m[3], m[4], p, grid, s);
    case EPI_SQRELU: return launch_tc<BN, STAGES, EPI_SQRELU>(m[0], m[1], m[2], m[3], m[4], p, grid, s);
    case EPI_GATE: return launch_tc<BN, STAGES, EPI_GATE>(m[0], m[1], m[2], m[3], m[4], p, grid, s);
    case EPI_ADD_RES: return launch_tc<BN, STAGES, EPI_ADD_RES>(m[0], m[1], m[2], m[3], m[4], p, grid, s);
    case EPI_PARTIAL: return launch_tc<BN, STAGES, EPI_PARTIAL>(m[0], m[1], m[2], m[3], m[4], p, grid, s);
    case EPI_SQRELU_Q8: return launch_tc<BN, STAGES, EPI_SQRELU_Q8>(m[0], m[1], m[2], m[3], m[4], p, grid, s);
    case EPI_SCALE: return launch_tc<BN, STAGES, EPI_SCALE>(m[0], m[1], m[2], m[3], m[4], p, grid, s);
  }
  return LMOE_ERR_INVALID_ARG;
}

lmoe_status tc_gemm(const TcLaunch& L, uint32_t* err_word, cudaStream_t stream) {
  const int bn = L.bn;
  if (bn != 32 && bn != 64 && bn != 128 && bn != 256) return LMOE_ERR_INVALID_ARG;
  // A always has 128-row boxes (activation rows normal, weight rows swap); B has BN-row boxes.
  // maps: A0, B0, A1, B1, and a 32-row token box of B0 for small weight-major tiles
  CUtensorMap maps[5];
  for (int sg = 0; sg < L.nseg; ++sg) {
    if (!make_map_bf16(&maps[2 * sg], L.a[sg], 128)) return LMOE_ERR_INVALID_ARG;
    if (!make_map_bf16(&maps[2 * sg + 1], L.b[sg], bn)) return LMOE_ERR_INVALID_ARG;
  }
  if (L.nseg == 1) {
    maps[2] = maps[0];
    maps[3] = maps[1];
  }
  if (L.swap && L.grouped && bn > 32) {
    if (!make_map_bf16(&maps[4], L.b[0], 32)) return LMOE_ERR_INVALID_ARG;
  } else {
    maps[4] = maps[1];
  }
  if (L.grouped && L.groups > 1024) return LMOE_ERR_UNSUPPORTED;
  if (L.grouped && !L.swap) return LMOE_ERR_INVALID_ARG;   // grouped tiles are weight-major
  TcParams p = {};
  p.swap = L.swap;
  p.grouped = L.grouped;
  p.rows = L.rows;
  p.cols = L.cols;
  p.nseg = L.nseg;
  for (int sg = 0; sg < 2; ++sg) {
    p.seg[sg].kblocks = L.kblocks[sg];
    p.seg[sg].a_kgroup = L.a_kgroup[sg];
    p.seg[sg].b_kgroup = L.b_kgroup[sg];
  }
  p.offsets = L.offsets;
  p.padded_offsets = L.padded_offsets;
  p.groups = L.groups;
  p.out = L.out;
  p.ld_out = L.ld_out;
  p.bias = L.bias;
  p.row_scale = L.row_scale;
  p.residual = static_cast<const __nv_bfloat16*>(L.residual);
  p.ld_res = L.ld_res;
  p.ksplit = L.ksplit > 1 ? L.ksplit : 1;
  p.partial = L.partial;
  p.fp8 = L.fp8;
  p.scale_a = L.scale_a;
  p.scale_w = L.scale_w;
  p.out_scale = L.out_scale;
  p.err = DevErr{err_word};
  for (int sg = 0; sg < L.nseg; ++sg)   // one operand kind per launch
    if (L.a[sg].elem != (L.fp8 ? 1 : 2) || L.b[sg].elem != (L.fp8 ? 1 : 2)) return LMOE_ERR_INVALID_ARG;
  if ((L.epi == EPI_SQRELU_Q8 && !L.out_scale) || ((L.epi == EPI_SQRELU_Q8 || L.epi == EPI_SCALE) && !L.fp8))
    return LMOE_ERR_INVALID_ARG;
  if (L.fp8 && L.grouped) return LMOE_ERR_UNSUPPORTED;
  if (p.ksplit > 1 && (L.grouped || !L.partial)) return LMOE_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  const int64_t tiles = L.max_tiles * p.ksplit;
  int64_t grid = tiles < sms ? tiles : sms;
  if (grid <= 0) return LMOE_OK;
  const int g = static_cast<int>(grid);
  const int epi = p.ksplit > 1 ? static_cast<int>(EPI_PARTIAL) : L.epi;
  lmoe_status st = LMOE_ERR_INVALID_ARG;
  switch (bn) {
    case 256: st = dispatch_epi<256, 4>(epi, maps, p, g, stream); break;
    case 128: st = dispatch_epi<128, 6>(epi, maps, p, g, stream); break;
    case 64: st = dispatch_epi<64, 8>(epi, maps, p, g, stream); break;
    case 32: st = dispatch_epi<32, 10>(epi, maps, p, g, stream); break;
  }
  if (st != LMOE_OK || p.ksplit == 1) return st;
  // deterministic reduction of the partial sums (fixed split order) + the real epilogue
  const int64_t n = static_cast<int64_t>(L.rows) * L.cols;
  int rblocks = static_cast<int>((n + 255) / 256);
  if (rblocks > sms * 8) rblocks = sms * 8;
  switch (L.epi) {
    case EPI_F32_BIAS: launch_k(splitk_reduce_kernel<EPI_F32_BIAS>, dim3(rblocks), dim3(256), 0, stream, p); break;
    case EPI_BF16: launch_k(splitk_reduce_kernel<EPI_BF16>, dim3(rblocks), dim3(256), 0, stream, p); break;
    case EPI_SQRELU: launch_k(splitk_reduce_kernel<EPI_SQRELU>, dim3(rblocks), dim3(256), 0, stream, p); break;
    case EPI_ADD_RES: launch_k(splitk_reduce_kernel<EPI_ADD_RES>, dim3(rblocks), dim3(256), 0, stream, p); break;
    case EPI_SQRELU_Q8: launch_k(splitk_reduce_kernel<EPI_SQRELU_Q8>, dim3(rblocks), dim3(256), 0, stream, p); break;
    case EPI_SCALE: launch_k(splitk_reduce_kernel<EPI_SCALE>, dim3(rblocks), dim3(256), 0, stream, p); break;
    default: return LMOE_ERR_INVALID_ARG;
  }
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

// ----- CTA-pair grouped GEMM (weight-major expert tiles) -----
template <int EPI>
static lmoe_status launch_tc2(const Tc2Maps& m, const TcParams& p, int64_t max_tiles, cudaStream_t s) {
  auto kern = tc2_gemm_kernel<EPI>;
  static std::atomic<uint64_t> configured{0};
  static std::atomic<int> max_clusters_dev[64];
  int dev = 0;
  cudaGetDevice(&dev);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = Tc2Smem::kBytes;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_clusters = 0;
  if (device_configured(configured, dev)) {
    max_clusters = max_clusters_dev[dev].load(std::memory_order_relaxed);
  } else {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tc2Smem::kBytes) != cudaSuccess)
      return LMOE_ERR_CUDA;
    cfg.gridDim = dim3(2 * (device_sm_count() / 2), 1, 1);
    if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess || max_clusters <= 0)
      return LMOE_ERR_CUDA;
    if (dev >= 0 && dev < 64) max_clusters_dev[dev].store(max_clusters, std::memory_order_relaxed);
    mark_configured(configured, dev);
  }
  const int64_t clusters = max_tiles < max_clusters ? max_tiles : max_clusters;
  if (clusters <= 0) return LMOE_OK;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  cfg.numAttrs = 2;   // cluster shape + programmatic serialisation (occupancy was queried with the shape only)
  if (cudaLaunchKernelEx(&cfg, kern, m, p) != cudaSuccess) return LMOE_ERR_CUDA;
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

lmoe_status tc2_gemm(const TcLaunch& L, uint32_t* err_word, cudaStream_t stream) {
  if (!L.swap || !L.grouped || L.nseg != 1 || L.ksplit > 1) return LMOE_ERR_INVALID_ARG;
  if (L.groups > Tc2Smem::kMaxGroups) return LMOE_ERR_UNSUPPORTED;
  // maps: weights (A, 128-row boxes), tokens (B) with 128/64/32/16-row boxes;
  // the same for the dense extra problem (copies of the first five without one)
  Tc2Maps maps;
  if (!make_map_bf16(&maps.m[0], L.a[0], 128)) return LMOE_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i)
    if (!make_map_bf16(&maps.m[1 + i], L.b[0], 128 >> i)) return LMOE_ERR_INVALID_ARG;
  const bool extra = L.rows_x > 0;
  if (extra) {
    if (L.cols_x <= 0) return LMOE_ERR_INVALID_ARG;
    if (L.x_kgroup > 0 ? (L.x_wt.k != L.x_kgroup || L.x_kgroup % 64 || L.x_act.k != L.x_kgroup * L.x_wt.groups)
                       : L.x_act.k != L.x_wt.k)
      return LMOE_ERR_INVALID_ARG;
    if (!make_map_bf16(&maps.m[5], L.x_wt, 128)) return LMOE_ERR_INVALID_ARG;
    for (int i = 0; i < 4; ++i)
      if (!make_map_bf16(&maps.m[6 + i], L.x_act, 128 >> i)) return LMOE_ERR_INVALID_ARG;
  } else {
    for (int i = 0; i < 5; ++i) maps.m[5 + i] = maps.m[i];
  }
  TcParams p = {};
  p.swap = 1;
  p.grouped = 1;
  p.rows = L.rows;
  p.cols = L.cols;
  p.nseg = 1;
  p.seg[0].kblocks = L.kblocks[0];
  p.offsets = L.offsets;
  p.padded_offsets = L.padded_offsets;
  p.groups = L.groups;
  p.out = L.out;
  p.ld_out = L.ld_out;
  p.row_scale = L.row_scale;
  p.ksplit = 1;
  p.rows_x = extra ? L.rows_x : 0;
  p.cols_x = extra ? L.cols_x : 0;
  p.kblocks_x = extra ? static_cast<int>((L.x_act.k + 63) / 64) : 0;
  p.kgroup_x = extra ? L.x_kgroup : 0;
  p.out_x = extra ? L.out_x : nullptr;
  p.ld_out_x = extra ? L.ld_out_x : 0;
  p.err = DevErr{err_word};
  const int64_t tiles = L.max_tiles + (extra ? ((L.rows_x + 255) / 256) * ((L.cols_x + 255) / 256) : 0);
  switch (L.epi) {
    case EPI_BF16: return launch_tc2<EPI_BF16>(maps, p, tiles, stream);
    case EPI_SQRELU: return launch_tc2<EPI_SQRELU>(maps, p, tiles, stream);
    case EPI_GATE: return launch_tc2<EPI_GATE>(maps, p, tiles, stream);
  }
  return LMOE_ERR_INVALID_ARG;
}

}  // namespace lmoe
