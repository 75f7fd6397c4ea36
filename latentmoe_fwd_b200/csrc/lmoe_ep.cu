// Expert parallelism in the latent dimension: the layout arithmetic of a
// dispatch/combine all-to-all over G ranks and the row-block reorder between
// the all-to-all's source-major order and the expert GEMMs' expert-grouped
// padded order. The greeksharifa page on the Nemotron 3 whitepaper (section
// 2.2 "LatentMoE") gives the reason to shard experts in l: the routed rows
// that cross GPUs are l-dim, so the all-to-all volume falls by d / l.
//
// Ownership: rank h owns the contiguous experts [first(h), first(h) + n(h)),
// n(h) = N / G, one more for the first N % G ranks.
// Send side (rank r): its permutation sorts slots by expert, so the rows for
// rank h are one contiguous block of its sorted rows.
// Receive side: the all-to-all delivers one block per source rank, in rank
// order, each sorted by expert; the expert GEMMs want every local expert's
// rows together (source rank ascending inside an expert) at padded offsets
// (multiples of 128), so each (source, expert) block moves as a whole.
#include <stdint.h>

#include "lmoe_device.cuh"
#include "lmoe_internal.h"

namespace lmoe {
namespace {

void ownership(int G, int N, int h, int* first, int* n) {
  const int base = N / G, extra = N % G;
  *first = h * base + (h < extra ? h : extra);
  *n = base + (h < extra ? 1 : 0);
}

// Copy row blocks: block b of `nblocks` moves count[b] rows from row src[b]
// of `in` to row dst[b] of `out` (rows of row_bytes, a multiple of 16).
// A warp per row, 16-byte accesses; blocks are found by a binary search over
// their inclusive row prefix.
__global__ void __launch_bounds__(256) ep_reorder_kernel(const uint8_t* __restrict__ in, uint8_t* __restrict__ out,
                                                         int64_t row_bytes, const int32_t* __restrict__ src,
                                                         const int32_t* __restrict__ dst,
                                                         const int64_t* __restrict__ prefix, int nblocks,
                                                         int64_t total) {
  pdl_begin();
  const int lane = threadIdx.x & 31;
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (r >= total) return;
  int lo = 0, hi = nblocks - 1;   // first block whose inclusive prefix exceeds r
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(prefix + mid) > r) hi = mid; else lo = mid + 1;
  }
  const int64_t start = lo > 0 ? __ldg(prefix + lo - 1) : 0;
  const int64_t i = r - start;
  const uint4* s = reinterpret_cast<const uint4*>(in + (static_cast<int64_t>(__ldg(src + lo)) + i) * row_bytes);
  uint4* d = reinterpret_cast<uint4*>(out + (static_cast<int64_t>(__ldg(dst + lo)) + i) * row_bytes);
  for (int64_t v = lane; v < row_bytes / 16; v += 32) d[v] = __ldg(s + v);
}

}  // namespace
}  // namespace lmoe

using namespace lmoe;

extern "C" {

lmoe_status lmoe_ep_plan(int G, int rank, int N, const int32_t* counts, int32_t* send_counts,
                         int32_t* send_offsets, int32_t* recv_counts, int32_t* recv_offsets, int32_t* first_expert,
                         int32_t* local_experts, int32_t* local_offsets, int32_t* local_padded_offsets,
                         int32_t* block_src, int32_t* block_dst, int32_t* block_rows) {
  if (G <= 0 || N <= 0 || rank < 0 || rank >= G || !counts || !send_counts || !send_offsets || !recv_counts ||
      !recv_offsets || !first_expert || !local_experts || !local_offsets || !local_padded_offsets || !block_src ||
      !block_dst || !block_rows)
    return LMOE_ERR_INVALID_ARG;
  if (N > 1024 || G > N) return LMOE_ERR_UNSUPPORTED;
  for (int64_t i = 0; i < static_cast<int64_t>(G) * N; ++i)
    if (counts[i] < 0) return LMOE_ERR_INVALID_ARG;
  int f0 = 0, nl = 0;
  ownership(G, N, rank, &f0, &nl);
  *first_expert = f0;
  *local_experts = nl;
  // send: rows of this rank for each owner, contiguous in its sorted order
  const int32_t* mine = counts + static_cast<int64_t>(rank) * N;
  int64_t run = 0;
  for (int h = 0; h < G; ++h) {
    int fh = 0, nh = 0;
    ownership(G, N, h, &fh, &nh);
    int64_t c = 0;
    for (int e = fh; e < fh + nh; ++e) c += mine[e];
    if (run + c > INT32_MAX) return LMOE_ERR_UNSUPPORTED;
    send_offsets[h] = static_cast<int32_t>(run);
    send_counts[h] = static_cast<int32_t>(c);
    run += c;
  }
  // receive: one block per source rank, in rank order
  run = 0;
  for (int g = 0; g < G; ++g) {
    int64_t c = 0;
    for (int e = f0; e < f0 + nl; ++e) c += counts[static_cast<int64_t>(g) * N + e];
    if (run + c > INT32_MAX) return LMOE_ERR_UNSUPPORTED;
    recv_offsets[g] = static_cast<int32_t>(run);
    recv_counts[g] = static_cast<int32_t>(c);
    run += c;
  }
  // local expert-grouped layout: rows of expert el from every source, padded to 128
  int64_t off = 0, poff = 0;
  for (int el = 0; el < nl; ++el) {
    int64_t tot = 0;
    for (int g = 0; g < G; ++g) tot += counts[static_cast<int64_t>(g) * N + f0 + el];
    local_offsets[el] = static_cast<int32_t>(off);
    local_padded_offsets[el] = static_cast<int32_t>(poff);
    off += tot;
    poff += (tot + 127) / 128 * 128;
    if (poff > INT32_MAX) return LMOE_ERR_UNSUPPORTED;
  }
  local_offsets[nl] = static_cast<int32_t>(off);
  local_padded_offsets[nl] = static_cast<int32_t>(poff);
  // blocks (source g, local expert el), source-major: where each sits in the
  // received buffer and where it goes in the expert-grouped buffer
  for (int g = 0; g < G; ++g) {
    int64_t src = recv_offsets[g];
    for (int el = 0; el < nl; ++el) {
      int64_t before = 0;
      for (int g2 = 0; g2 < g; ++g2) before += counts[static_cast<int64_t>(g2) * N + f0 + el];
      const int64_t b = static_cast<int64_t>(g) * nl + el;
      const int32_t c = counts[static_cast<int64_t>(g) * N + f0 + el];
      block_src[b] = static_cast<int32_t>(src);
      block_dst[b] = static_cast<int32_t>(local_padded_offsets[el] + before);
      block_rows[b] = c;
      src += c;
    }
  }
  return LMOE_OK;
}

lmoe_status lmoe_ep_reorder(const void* in, void* out, int64_t row_bytes, int nblocks, const int32_t* src_rows,
                            const int32_t* dst_rows, const int64_t* row_prefix, int64_t total_rows, void* stream) {
  if (total_rows < 0 || nblocks < 0) return LMOE_ERR_INVALID_ARG;
  if (total_rows == 0) return LMOE_OK;
  if (!in || !out || !src_rows || !dst_rows || !row_prefix || nblocks == 0) return LMOE_ERR_INVALID_ARG;
  if (row_bytes <= 0 || row_bytes % 16 || (reinterpret_cast<uintptr_t>(in) & 15) ||
      (reinterpret_cast<uintptr_t>(out) & 15))
    return LMOE_ERR_INVALID_ARG;
  const int64_t blocks = (total_rows * 32 + 255) / 256;
  if (blocks > 0x7fffffff) return LMOE_ERR_UNSUPPORTED;
  launch_k(ep_reorder_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, static_cast<cudaStream_t>(stream),
           static_cast<const uint8_t*>(in), static_cast<uint8_t*>(out), row_bytes, src_rows, dst_rows, row_prefix,
           nblocks, total_rows);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

}  // extern "C"
