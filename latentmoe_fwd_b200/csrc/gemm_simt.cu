// fp32 GEMM on the CUDA cores for fp32 layers (no tensor-core fp32 path):
//   out[row, col] = epi( sum_k A[row, k] * B[g][col, k] )
// 64 x 64 output tiles, 256 threads with 4 x 4 outputs each, 16-wide K slices
// staged in shared memory. Grouped mode reads the expert of each 128-row
// padded tile from the padded offsets, like the tensor-core kernel.
#include "gemm_tc.cuh"   // EpiKind
#include "lmoe_internal.h"

namespace lmoe {

constexpr int kST = 64;   // tile edge
constexpr int kSK = 16;   // K slice

__device__ __forceinline__ float simt_epi(int epi, float acc, const SimtLaunch& p, int64_t row, int col) {
  switch (epi) {
    case EPI_SQRELU: {
      const float r = fmaxf(acc, 0.0f);
      return r * r;
    }
    case EPI_GATE: return p.row_scale ? acc * p.row_scale[row] : acc;
    case EPI_F32_BIAS: return p.bias ? acc + p.bias[col] : acc;
    case EPI_ADD_RES: return acc + p.residual[row * p.ld_res + col];
  }
  return acc;
}

__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtLaunch p) {
  pdl_begin();
  __shared__ float sa[kSK][kST + 1];
  __shared__ float sb[kSK][kST + 1];
  const int64_t row0 = static_cast<int64_t>(blockIdx.y) * kST;
  const int col0 = blockIdx.x * kST;
  int g = 0;
  int64_t row_end = p.rows;
  if (p.grouped) {
    if (row0 >= p.padded_offsets[p.groups]) return;
    // expert owning the 128-row tile that contains row0
    int lo = 0, hi = p.groups;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.padded_offsets[mid] <= row0) lo = mid; else hi = mid - 1;
    }
    g = lo;
    row_end = p.padded_offsets[g] + (p.offsets[g + 1] - p.offsets[g]);
    if (row0 >= row_end) return;
  }
  const float* B = p.b + static_cast<int64_t>(g) * p.cols * p.k;
  const int64_t lda = p.lda ? p.lda : p.k;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < p.k; k0 += kSK) {
    for (int i = threadIdx.x; i < kSK * kST; i += 256) {
      const int kk = i % kSK, rr = i / kSK;
      const int64_t ar = row0 + rr;
      const int bc = col0 + rr;
      sa[kk][rr] = (ar < row_end && k0 + kk < p.k) ? p.a[ar * lda + k0 + kk] : 0.0f;
      sb[kk][rr] = (bc < p.cols && k0 + kk < p.k) ? B[static_cast<int64_t>(bc) * p.k + k0 + kk] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = sa[kk][ty * 4 + i];
        bv[i] = sb[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = row0 + ty * 4 + i;
    if (row >= row_end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = col0 + tx * 4 + j;
      if (col >= p.cols) continue;
      float v = acc[i][j];
      if (p.accumulate) v += p.out[row * p.ld_out + col];
      p.out[row * p.ld_out + col] = simt_epi(p.epi, v, p, row, col);
    }
  }
}

lmoe_status simt_gemm(const SimtLaunch& L, uint32_t* err_word, cudaStream_t stream) {
  (void)err_word;
  if (L.rows <= 0 || L.cols <= 0) return LMOE_OK;
  dim3 grid((L.cols + kST - 1) / kST, (L.rows + kST - 1) / kST);
  launch_k(simt_gemm_kernel, dim3(grid), dim3(256), 0, stream, L);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

}  // namespace lmoe
