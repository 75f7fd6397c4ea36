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
// Peer-memory data plane: instead of an all-to-all and a reorder, each rank's
// dispatch kernel stores its rows straight at their final rows in the owners'
// buffers (the owner's padded row of this rank's first row for the expert,
// plus the slot's rank within the expert here), and its combine kernel reads
// the owners' expert outputs back from the same rows. Plain loads and stores
// through the peers' pointers: no TMA and no multicast touch another GPU.
#include <cuda_bf16.h>
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

// Dispatch over peer memory: a warp per token reads its row once (2 KB per
// pass, four 16-byte loads per lane) and stores it, with its gate, at each of
// its K slots' rows in the owner rank's expert-grouped buffer. Slot f = t*K+k
// of expert e goes to rank owner[e], row dst_base[e] + inv_perm[f] - offsets[e].
// Plain stores to peer-mapped (or local) memory; a slot whose expert or row is
// out of range is skipped and reported.
__global__ void __launch_bounds__(256) ep_dispatch_kernel(
    const uint8_t* __restrict__ rows, int64_t T, int64_t row_bytes, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ inv_perm, const int32_t* __restrict__ offsets, const int32_t* __restrict__ owner,
    const int32_t* __restrict__ dst_base, uint8_t* const* __restrict__ peer_rows, const float* __restrict__ gates,
    float* const* __restrict__ peer_gates, int K, int N, int G, int64_t rows_cap, DevErr err) {
  pdl_begin();
  constexpr unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int64_t n16 = row_bytes >> 4;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    int h = -1;
    int64_t row = -1;
    if (lane < K) {
      const int64_t f = t * K + lane;
      const int e = __ldg(idx + f);
      if (e >= 0 && e < N) {
        h = __ldg(owner + e);
        row = static_cast<int64_t>(__ldg(dst_base + e)) + __ldg(inv_perm + f) - __ldg(offsets + e);
        // a rank, row or buffer (16-byte stores) out of range is skipped and reported
        if (h < 0 || h >= G || row < 0 || row >= rows_cap || (reinterpret_cast<uintptr_t>(peer_rows[h]) & 15)) {
          dev_report(err, kErrBounds, static_cast<uint32_t>(f));
          h = -1;
        }
      }
      if (h >= 0 && gates && peer_gates) peer_gates[h][row] = __ldg(gates + f);
    }
    const uint4* src = reinterpret_cast<const uint4*>(rows + t * row_bytes);
    for (int64_t i0 = 0; i0 < n16; i0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i = i0 + u * 32 + lane;
        v[u] = i < n16 ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
      }
      for (int k = 0; k < K; ++k) {
        const int hk = __shfl_sync(FULL, h, k);
        const int64_t rk = __shfl_sync(FULL, row, k);
        if (hk < 0) continue;
        uint4* dst = reinterpret_cast<uint4*>(peer_rows[hk] + rk * row_bytes);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t i = i0 + u * 32 + lane;
          if (i < n16) dst[i] = v[u];
        }
      }
    }
  }
}

// Combine over peer memory: c[t] = sum over the token's in-range slots, in k
// order, of the owner's y row (gates already applied by the owner), in fp32,
// stored BF16 -- the arithmetic of the single-GPU combine with no gate. A CTA
// per token.
__global__ void __launch_bounds__(256) ep_combine_kernel(
    const __nv_bfloat16* const* __restrict__ peer_y, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ inv_perm, const int32_t* __restrict__ offsets, const int32_t* __restrict__ owner,
    const int32_t* __restrict__ dst_base, __nv_bfloat16* __restrict__ c, int K, int N, int G, int l,
    int64_t rows_cap, DevErr err) {
  pdl_begin();
  __shared__ const __nv_bfloat16* rowp[32];
  __shared__ int s_nk;
  const int64_t t = blockIdx.x;
  if (threadIdx.x < 32) {
    const int k = threadIdx.x;
    bool ok = false;
    const __nv_bfloat16* p = nullptr;
    if (k < K) {
      const int64_t f = t * K + k;
      const int e = __ldg(idx + f);
      if (e >= 0 && e < N) {
        const int h = __ldg(owner + e);
        const int64_t row = static_cast<int64_t>(__ldg(dst_base + e)) + __ldg(inv_perm + f) - __ldg(offsets + e);
        ok = h >= 0 && h < G && row >= 0 && row < rows_cap && !(reinterpret_cast<uintptr_t>(peer_y[h]) & 15);
        if (ok) p = peer_y[h] + row * l;
        else dev_report(err, kErrBounds, static_cast<uint32_t>(f));
      }
    }
    const unsigned m = __ballot_sync(0xffffffffu, ok);
    if (ok) rowp[__popc(m & ((1u << k) - 1u))] = p;
    if (k == 0) s_nk = __popc(m);
  }
  __syncthreads();
  const int nk = s_nk;
  for (int col = threadIdx.x * 8; col < l; col += blockDim.x * 8) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int k = 0; k < nk; ++k) {
      const uint4 u = *reinterpret_cast<const uint4*>(rowp[k] + col);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f2 = __bfloat1622float2(h2[i]);
        acc[2 * i] += f2.x;
        acc[2 * i + 1] += f2.y;
      }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(c + t * l + col) = o;
  }
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

lmoe_status lmoe_ep_slot_bases(int G, int rank, int N, const int32_t* counts, int32_t* expert_owner,
                               int32_t* dst_base) {
  if (G <= 0 || N <= 0 || rank < 0 || rank >= G || !counts || !expert_owner || !dst_base)
    return LMOE_ERR_INVALID_ARG;
  if (N > 1024 || G > N) return LMOE_ERR_UNSUPPORTED;
  for (int64_t i = 0; i < static_cast<int64_t>(G) * N; ++i)
    if (counts[i] < 0) return LMOE_ERR_INVALID_ARG;
  for (int h = 0; h < G; ++h) {
    int f0 = 0, nl = 0;
    ownership(G, N, h, &f0, &nl);
    int64_t poff = 0;   // owner h's padded offset of its expert f0 + el
    for (int el = 0; el < nl; ++el) {
      const int e = f0 + el;
      int64_t tot = 0, before = 0;
      for (int g = 0; g < G; ++g) {
        const int64_t c = counts[static_cast<int64_t>(g) * N + e];
        tot += c;
        if (g < rank) before += c;
      }
      if (poff + before > INT32_MAX) return LMOE_ERR_UNSUPPORTED;
      expert_owner[e] = h;
      dst_base[e] = static_cast<int32_t>(poff + before);
      poff += (tot + 127) / 128 * 128;
    }
  }
  return LMOE_OK;
}

lmoe_status lmoe_ep_dispatch(int64_t T, int K, int N, int G, const void* rows, int64_t row_bytes,
                             const int32_t* topk_idx, const int32_t* inv_perm, const int32_t* offsets,
                             const int32_t* expert_owner, const int32_t* dst_base, void* const* peer_rows,
                             int64_t peer_rows_cap, const float* topk_w, float* const* peer_gates, uint32_t* err_word,
                             void* stream) {
  if (T < 0 || K < 1 || K > 32 || N < 1 || G < 1 || peer_rows_cap < 0) return LMOE_ERR_INVALID_ARG;
  if (T == 0) return LMOE_OK;
  if (!rows || !topk_idx || !inv_perm || !offsets || !expert_owner || !dst_base || !peer_rows)
    return LMOE_ERR_INVALID_ARG;
  if (row_bytes <= 0 || row_bytes % 16 || (reinterpret_cast<uintptr_t>(rows) & 15)) return LMOE_ERR_INVALID_ARG;
  if ((topk_w == nullptr) != (peer_gates == nullptr)) return LMOE_ERR_INVALID_ARG;
  const int64_t sms = device_sm_count();
  int64_t blocks = (T * 32 + 255) / 256;
  if (blocks > sms * 8) blocks = sms * 8;
  launch_k(ep_dispatch_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, static_cast<cudaStream_t>(stream),
           static_cast<const uint8_t*>(rows), T, row_bytes, topk_idx, inv_perm, offsets, expert_owner, dst_base,
           reinterpret_cast<uint8_t* const*>(peer_rows), topk_w, peer_gates, K, N, G, peer_rows_cap,
           DevErr{err_word});
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

lmoe_status lmoe_ep_combine(int64_t T, int K, int N, int G, int l, const void* const* peer_y, int64_t peer_rows_cap,
                            const int32_t* topk_idx, const int32_t* inv_perm, const int32_t* offsets,
                            const int32_t* expert_owner, const int32_t* dst_base, void* c, uint32_t* err_word,
                            void* stream) {
  if (T < 0 || K < 1 || K > 32 || N < 1 || G < 1 || l <= 0 || l % 8 || peer_rows_cap < 0)
    return LMOE_ERR_INVALID_ARG;
  if (T == 0) return LMOE_OK;
  if (!peer_y || !topk_idx || !inv_perm || !offsets || !expert_owner || !dst_base || !c) return LMOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(c) & 15) return LMOE_ERR_INVALID_ARG;
  if (T > 0x7fffffff) return LMOE_ERR_UNSUPPORTED;
  launch_k(ep_combine_kernel, dim3(static_cast<unsigned>(T)), dim3(256), 0, static_cast<cudaStream_t>(stream),
           reinterpret_cast<const __nv_bfloat16* const*>(peer_y), topk_idx, inv_perm, offsets, expert_owner,
           dst_base, static_cast<__nv_bfloat16*>(c), K, N, G, l, peer_rows_cap, DevErr{err_word});
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

}  // extern "C"
