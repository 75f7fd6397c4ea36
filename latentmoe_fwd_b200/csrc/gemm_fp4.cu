// Host side of the grouped NVFP4 expert GEMM: tensor maps over packed E2M1
// codes and the launch of the two epilogue variants.
#include <mutex>

#include "gemm_fp4.cuh"
#include "gemm_tc.cuh"
#include "lmoe_internal.h"

namespace lmoe {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn_fp4() {
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

// 3-D map over packed codes [groups][rows][k/2 bytes]; box 128 B x box_rows, 128-byte swizzle.
static bool make_map_fp4(CUtensorMap* map, const void* ptr, int64_t k, int64_t rows, int64_t groups,
                         int box_rows) {
  EncodeTiledFn enc = encode_fn_fp4();
  if (!enc || !ptr || (reinterpret_cast<uintptr_t>(ptr) & 15) || (k / 2) % 16) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(k / 2), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(groups)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(k / 2), static_cast<cuuint64_t>(rows * (k / 2))};
  cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, bool BATCH = false>
static lmoe_status launch_fp4(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a32, const Fp4Params& p,
                              int grid, cudaStream_t s) {
  auto kern = fp4_gemm_kernel<EPI, BATCH>;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!device_configured(configured, dev)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Fp4Smem::kBytes) != cudaSuccess)
      return LMOE_ERR_CUDA;
    mark_configured(configured, dev);
  }
  launch_k(kern, dim3(grid), dim3(Fp4Smem::kThreads), Fp4Smem::kBytes, s, a, b, a32, p);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

lmoe_status fp4_gemm(const Fp4Launch& L, uint32_t* err_word, cudaStream_t stream) {
  if (L.k % 256 || L.cols % 256 || L.groups > Fp4Smem::kMaxGroups) return LMOE_ERR_UNSUPPORTED;
  const bool batch = L.kgroups != nullptr;
  if (batch && (L.quant_out || L.f32_out || L.row_scale || L.a_rows % 128 || L.groups < 1)) return LMOE_ERR_UNSUPPORTED;
  CUtensorMap ma, mb;
  CUtensorMap ma32;   // 32-row boxes for tiles with at most 32 real rows
  if (!make_map_fp4(&ma, L.a_codes, L.k, L.a_rows, 1, 128)) return LMOE_ERR_INVALID_ARG;
  if (!make_map_fp4(&ma32, L.a_codes, L.k, L.a_rows, 1, 32)) return LMOE_ERR_INVALID_ARG;
  if (!make_map_fp4(&mb, L.b_codes, L.k, L.cols, batch ? 1 : L.groups, 256)) return LMOE_ERR_INVALID_ARG;
  Fp4Params p;
  p.rows = static_cast<int>(L.a_rows);
  p.cols = L.cols;
  p.kblocks = static_cast<int>(L.k / 256);
  p.sf_groups_a = static_cast<int>(L.k / 64);
  p.sf_groups_b = static_cast<int>(L.k / 64);
  p.sfa = L.a_sf;
  p.sfb = L.b_sf;
  p.sfb_expert_bytes = batch ? 0 : static_cast<long long>(L.cols) * (L.k / 16);
  p.kgroup_tab = L.kgroups;
  p.out_group_stride = L.out_group_stride;
  p.offsets = L.offsets;
  p.padded_offsets = L.padded_offsets;
  p.groups = L.groups;
  p.in_scale = L.in_scale;
  p.in_scale_grouped = L.in_scale_grouped;
  p.w_scale = L.w_scale;
  p.out_scale = L.out_scale;
  p.row_scale = L.row_scale;
  p.out = L.out;
  p.out_sf = L.out_sf;
  p.ld_out = L.ld_out;
  p.out_vec32 = (reinterpret_cast<uintptr_t>(L.out) % 32 == 0) && (L.ld_out * 2) % 32 == 0;
  if (L.f32_out && ((reinterpret_cast<uintptr_t>(L.out) & 15) || L.ld_out % 4)) return LMOE_ERR_INVALID_ARG;
  p.err = DevErr{err_word};
  const int sms = device_sm_count();
  const int64_t tiles = (L.a_rows / 128) * (L.cols / 256) * (batch ? L.groups : 1);
  if (tiles > 0x7fffffff) return LMOE_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  if (grid <= 0) return LMOE_OK;
  if (batch) return launch_fp4<FP4_EPI_GATE_BF16, true>(ma, mb, ma32, p, grid, stream);
  if (L.quant_out) return launch_fp4<FP4_EPI_SQRELU_QUANT>(ma, mb, ma32, p, grid, stream);
  if (L.f32_out) return launch_fp4<FP4_EPI_F32>(ma, mb, ma32, p, grid, stream);
  return launch_fp4<FP4_EPI_GATE_BF16>(ma, mb, ma32, p, grid, stream);
}

}  // namespace lmoe
