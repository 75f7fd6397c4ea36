// Router top-K, expert-grouped permutation, gather, combine and the NVFP4
// quantiser. These steps are bound by memory latency or bandwidth, not by
// arithmetic: they use coalesced 16-byte accesses, warp intrinsics and
// shared memory, and no global atomics in the data path.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "lmoe_device.cuh"
#include "lmoe_internal.h"

namespace lmoe {

// ===========================================================================
// Top-K + renormalised softmax gates.
// Selection order: logit descending, expert index ascending (ties to the
// lower index). Gates: exp(l_k - l_max) / sum over the K chosen.
//
// Exact decisions from approximate logits: tensor-core logits carry fp32
// accumulation error. When the kernel is given x and W_r, every adjacent pair
// among the K+1 largest logits (and any further expert near the K-th) whose
// gap is within 2*tau gets its logits recomputed exactly, and the candidates
// are re-ranked. Experts left approximate are more than 2*tau from every
// neighbour, so their order is exact as long as the logit error is below
// tau. tau scales with the token's bias-free logit RMS (the size of the
// GEMM's partial sums): tau = 2^-12 * RMS + 2^-22 * max|logit|. The GEMM adds
// d/16 MMA results into an fp32 accumulator, each addition off by at most
// 2^-24 (2^-23 if truncated) of a partial sum, and the partial sums of a
// random-signed dot stay near the logit's own size: 512 steps (d = 8192)
// give 2^-15 to 2^-14 of the RMS, a quarter or less of tau. The largest error
// measured on the Zipf-biased d = 8192 layer is 0.22 tau. Every candidate
// inside the window costs one exact d-long dot, so the window is kept narrow.
//
// Work split: a block of eight warps owns `tpb` tokens (eight, or one when
// there are few tokens). A token's warp extracts its candidates; the exact
// dot products of all of the block's marked candidates then form one pool
// that every warp of the block draws from, each dot split over up to eight
// warps when the pool is small, so a decode batch of a few tokens does not
// run its dots one after another on one warp.
// ===========================================================================
constexpr int kTopkWarps = 8;
constexpr int kTopkPieces = kTopkWarps * 32;

// Exact logit pieces. Products of two BF16 (or the fp32 layer's fp32) values
// are formed exactly where the format allows and summed as an unevaluated
// fp32 pair (hi, lo) with error-free TwoSum steps, so the result carries ~48
// significant bits -- without fp64 arithmetic, which is slow on this part.
__device__ __forceinline__ void two_sum_acc(float& hi, float& lo, float p) {
  const float s = __fadd_rn(hi, p);
  const float bb = __fsub_rn(s, hi);
  const float err = __fadd_rn(__fsub_rn(hi, __fsub_rn(s, bb)), __fsub_rn(p, bb));
  hi = s;
  lo = __fadd_rn(lo, err);
}

template <typename TA>
__device__ __forceinline__ void dot_vec(const uint4& a, const uint4& b, float& hi, float& lo) {
  if constexpr (sizeof(TA) == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 fa = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(&a)[i]);
      const float2 fb = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(&b)[i]);
      two_sum_acc(hi, lo, __fmul_rn(fa.x, fb.x));   // exact: 8 x 8 significant bits
      two_sum_acc(hi, lo, __fmul_rn(fa.y, fb.y));
    }
  } else {
    const float* fa = reinterpret_cast<const float*>(&a);
    const float* fb = reinterpret_cast<const float*>(&b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float p = __fmul_rn(fa[i], fb[i]);
      two_sum_acc(hi, lo, p);
      lo = __fadd_rn(lo, fmaf(fa[i], fb[i], -p));   // the product's own rounding error
    }
  }
}

// Double-word sum of x[j] * w[j] over j in [j0, j1) (multiples of the 16-byte
// vector), reduced over the warp. Eight 16-byte loads of each operand are in
// flight per lane; two accumulator pairs shorten the dependency chain.
template <typename TA>
__device__ __forceinline__ float2 exact_dot_range(const TA* __restrict__ x, const TA* __restrict__ w, int j0, int j1,
                                                  int lane) {
  constexpr int V = 16 / sizeof(TA);   // elements per 16-byte vector
  float hi0 = 0.0f, lo0 = 0.0f, hi1 = 0.0f, lo1 = 0.0f;
  int j = j0 + lane * V;
  for (; j + 7 * 32 * V < j1; j += 8 * 32 * V) {
    uint4 a[8], b[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      a[u] = __ldg(reinterpret_cast<const uint4*>(x + j + u * 32 * V));
      b[u] = __ldg(reinterpret_cast<const uint4*>(w + j + u * 32 * V));
    }
#pragma unroll
    for (int u = 0; u < 8; u += 2) {
      dot_vec<TA>(a[u], b[u], hi0, lo0);
      dot_vec<TA>(a[u + 1], b[u + 1], hi1, lo1);
    }
  }
  for (; j < j1; j += 32 * V)   // remainder, one vector at a time
    dot_vec<TA>(__ldg(reinterpret_cast<const uint4*>(x + j)), __ldg(reinterpret_cast<const uint4*>(w + j)), hi0, lo0);
  two_sum_acc(hi0, lo0, hi1);
  lo0 = __fadd_rn(lo0, lo1);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ohi = __shfl_xor_sync(0xffffffffu, hi0, off);
    const float olo = __shfl_xor_sync(0xffffffffu, lo0, off);
    two_sum_acc(hi0, lo0, ohi);
    lo0 = __fadd_rn(lo0, olo);
  }
  return make_float2(hi0, lo0);
}

// (value desc, index asc) ordering
__device__ __forceinline__ bool before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Unsigned key with the order of the float (-0 and +0 equal); 0 marks
// "nothing", NaN sorts below every number.
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 1u;
  if (f == 0.0f) return 0x80000000u;
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// The float an order key came from (+0 for either zero, a NaN for 1u).
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

template <int NPL, typename TA>
__global__ void __launch_bounds__(kTopkWarps * 32) topk_kernel(const float* __restrict__ logits, int64_t T, int N,
                                                               int K, int tpb, int32_t* __restrict__ idx,
                                                               float* __restrict__ w, const TA* __restrict__ x,
                                                               const TA* __restrict__ wr,
                                                               const float* __restrict__ bias, int d,
                                                               int refine_all) {
  pdl_begin();
  __shared__ int s_njobs[kTopkWarps];
  __shared__ int s_expert[kTopkWarps * 32];
  __shared__ float2 s_part[kTopkPieces];
  constexpr unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * tpb + warp;
  const bool has_token = warp < tpb && t < T;
  const bool refine = x != nullptr;

  float my_v = -INFINITY;   // lane c holds candidate c
  int my_i = 0x7fffffff;
  int C = 0;
  unsigned todo = 0;
  if (has_token) {
    const float* row = logits + t * N;
    float v[NPL];
    uint32_t key[NPL];
    float sq = 0.0f, vmax_abs = 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int col = lane + 32 * i;
      v[i] = col < N ? __ldg(row + col) : -INFINITY;
      key[i] = col < N ? order_key(v[i]) : 0u;
      if (col < N) {
        const float nb = v[i] - (bias ? __ldg(bias + col) : 0.0f);
        sq = fmaf(nb, nb, sq);
        vmax_abs = fmaxf(vmax_abs, fabsf(v[i]));
      }
    }
    float tau = 0.0f;
    if (refine) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        sq += __shfl_xor_sync(FULL, sq, off);
        vmax_abs = fmaxf(vmax_abs, __shfl_xor_sync(FULL, vmax_abs, off));
      }
      tau = ldexpf(sqrtf(sq / static_cast<float>(N)), -12) + ldexpf(vmax_abs, -22);
    }
    // this lane's four best remaining entries, best first (largest key; the
    // lower column first among equal keys); a lane that wins passes on to its
    // next one and scans its entries again only when all four are gone
    uint32_t taken = 0;
    uint32_t bk[4];
    int bi[4];
    auto rebuild = [&]() {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bk[j] = 0u;
        bi[j] = 0;
      }
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const uint32_t ki = ((taken >> i) & 1u) ? 0u : key[i];
        if (ki > bk[3]) {   // strictly greater: an equal key stays behind the lower column
          if (ki > bk[2]) {
            bk[3] = bk[2];
            bi[3] = bi[2];
            if (ki > bk[1]) {
              bk[2] = bk[1];
              bi[2] = bi[1];
              if (ki > bk[0]) {
                bk[1] = bk[0];
                bi[1] = bi[0];
                bk[0] = ki;
                bi[0] = i;
              } else {
                bk[1] = ki;
                bi[1] = i;
              }
            } else {
              bk[2] = ki;
              bi[2] = i;
            }
          } else {
            bk[3] = ki;
            bi[3] = i;
          }
        }
      }
    };
    rebuild();
    // extract candidates in (approximate) order: the K best, the (K+1)-th, and
    // while refining, further experts within 2 tau of the K-th (at most 32)
    float kth = -INFINITY;
    const int cmax = min(N, 32);
    while (C < cmax) {
      const uint32_t mk = __reduce_max_sync(FULL, bk[0]);
      if (mk == 0u) break;
      const unsigned bal = __ballot_sync(FULL, bk[0] == mk);
      int wl = __ffs(bal) - 1;
      if (bal & (bal - 1u))   // equal values in several lanes: the lowest column wins
        wl = static_cast<int>(__reduce_min_sync(FULL, bk[0] == mk ? static_cast<uint32_t>(bi[0] * 32 + lane) : ~0u) &
                              31u);
      const float bv = key_value(mk);
      const int bidx = __shfl_sync(FULL, bi[0] * 32 + lane, wl);
      if (C >= K && !(refine && bv >= kth - 2.0f * tau)) break;   // not a boundary candidate
      if (lane == C) {
        my_v = bv;
        my_i = bidx;
      }
      if (C == K - 1) kth = bv;
      ++C;
      if (!refine && C >= K) break;
      if (lane == wl) {   // the winning lane moves on to its next entry
        taken |= 1u << bi[0];
        bk[0] = bk[1];
        bi[0] = bi[1];
        bk[1] = bk[2];
        bi[1] = bi[2];
        bk[2] = bk[3];
        bi[2] = bi[3];
        bk[3] = 0u;
        if (bk[0] == 0u) rebuild();
      }
    }
    if (refine) {
      // mark candidates that have a neighbour within 2 tau (every candidate
      // with refine_all: exact logits, hence gates to fp32 rounding)
      const float up = __shfl_up_sync(FULL, my_v, 1);
      const float dn = __shfl_down_sync(FULL, my_v, 1);
      const bool mark = lane < C && (refine_all || (lane > 0 && up - my_v <= 2.0f * tau) ||
                                     (lane + 1 < C && my_v - dn <= 2.0f * tau));
      todo = __ballot_sync(FULL, mark);
      if (mark) s_expert[warp * 32 + __popc(todo & ((1u << lane) - 1u))] = my_i;
    }
  }
  if (refine) {
    // pooled exact dots: jobs numbered in warp order, each split into nseg pieces
    if (lane == 0) s_njobs[warp] = has_token ? __popc(todo) : 0;
    __syncthreads();
    const int nj = lane < kTopkWarps ? s_njobs[lane] : 0;
    int incl = nj;
#pragma unroll
    for (int off = 1; off < kTopkWarps; off <<= 1) {
      const int o = __shfl_up_sync(FULL, incl, off);
      if (lane >= off) incl += o;
    }
    const int total = __shfl_sync(FULL, incl, kTopkWarps - 1);
    if (total > 0) {
      const int nseg = total >= kTopkWarps ? 1 : kTopkWarps / total;
      constexpr int V = 16 / sizeof(TA);
      const int chunk = ((d / V + nseg - 1) / nseg) * V;
      for (int pc = warp; pc < total * nseg; pc += kTopkWarps) {
        const int job = pc / nseg;
        const int seg = pc - job * nseg;
        const int ow = __popc(__ballot_sync(FULL, lane < kTopkWarps && incl <= job));   // owning warp
        const int excl = __shfl_sync(FULL, incl - nj, ow);
        const int e = s_expert[ow * 32 + (job - excl)];
        const int64_t tok = static_cast<int64_t>(blockIdx.x) * tpb + ow;
        const int j0 = min(d, seg * chunk);
        const int j1 = min(d, j0 + chunk);
        const float2 r = exact_dot_range<TA>(x + tok * d, wr + static_cast<int64_t>(e) * d, j0, j1, lane);
        if (lane == 0) s_part[pc] = r;
      }
      __syncthreads();
      const int my_excl = __shfl_sync(FULL, incl - nj, warp);
      if ((todo >> lane) & 1u) {
        const int job = my_excl + __popc(todo & ((1u << lane) - 1u));
        float hi = 0.0f, lo = 0.0f;
        for (int sg = 0; sg < nseg; ++sg) {
          const float2 r = s_part[job * nseg + sg];
          two_sum_acc(hi, lo, r.x);
          lo = __fadd_rn(lo, r.y);
        }
        double val = static_cast<double>(hi) + static_cast<double>(lo);
        if (bias) val += static_cast<double>(__ldg(bias + my_i));
        my_v = static_cast<float>(val);
      }
    }
  }
  if (!has_token) return;
  // rank of each candidate among the C: the extraction order, unless the
  // exact refinement changed some of the values
  int rank = lane;
  if (todo != 0u) {
    rank = 0;
    for (int c = 0; c < C; ++c) {
      const float ov = __shfl_sync(FULL, my_v, c);
      const int oi = __shfl_sync(FULL, my_i, c);
      if (lane < C && c != lane && before(ov, oi, my_v, my_i)) ++rank;
    }
  }
  const bool chosen = lane < C && rank < K;
  // the largest logit is rank 0
  const unsigned top_mask = __ballot_sync(FULL, lane < C && rank == 0);
  const float lmax = __shfl_sync(FULL, my_v, __ffs(top_mask) - 1);
  const float e = chosen ? expf(my_v - lmax) : 0.0f;
  float sum = e;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL, sum, off);
  if (chosen) {
    idx[t * K + rank] = my_i;
    w[t * K + rank] = __fdiv_rn(e, sum);
  }
}

lmoe_status launch_topk(const float* logits, int64_t T, int N, int K, int32_t* idx, float* w, const void* x,
                        const void* w_router, const float* bias, int d, int act, uint32_t* err, cudaStream_t s,
                        int refine_all) {
  (void)err;
  if (T == 0) return LMOE_OK;
  // few tokens: one token per block, so the block's eight warps share its dots
  const int tpb = (x != nullptr && T <= 1024) ? 1 : kTopkWarps;
  const int64_t blocks64 = (T + tpb - 1) / tpb;
  if (blocks64 > 0x7fffffff) return LMOE_ERR_UNSUPPORTED;
  const int blocks = static_cast<int>(blocks64);
  const int npl = (N + 31) / 32;
#define LMOE_TOPK(NPLV)                                                                                       \
  do {                                                                                                       \
    if (act == LMOE_F32)                                                                                     \
      launch_k(topk_kernel<NPLV, float>, dim3(blocks), dim3(kTopkWarps * 32), 0, s, logits, T, N, K, tpb, idx, \
               w, static_cast<const float*>(x), static_cast<const float*>(w_router), bias, d, refine_all);   \
    else                                                                                                     \
      launch_k(topk_kernel<NPLV, __nv_bfloat16>, dim3(blocks), dim3(kTopkWarps * 32), 0, s, logits, T, N, K,   \
               tpb, idx, w, static_cast<const __nv_bfloat16*>(x),                                            \
               static_cast<const __nv_bfloat16*>(w_router), bias, d, refine_all);                            \
  } while (0)
  if (npl <= 1) LMOE_TOPK(1);
  else if (npl <= 2) LMOE_TOPK(2);
  else if (npl <= 4) LMOE_TOPK(4);
  else if (npl <= 8) LMOE_TOPK(8);
  else if (npl <= 16) LMOE_TOPK(16);
  else if (npl <= 32) LMOE_TOPK(32);
  else return LMOE_ERR_UNSUPPORTED;
#undef LMOE_TOPK
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

// ===========================================================================
// Permutation: stable counting sort of slots f = t*K + k by expert.
//   pass 1 (count):  per chunk of slots, a shared-memory histogram, stored
//                    expert-major: cnt[e * nchunks + chunk].
//   pass 2 (scan):   a warp per expert turns its row of chunk counts into
//                    exclusive prefixes (coalesced, 32 chunks per step) and
//                    stores the expert's total at cnt[N * nchunks + e].
//   pass 3 (scatter): every CTA first scans the N totals in shared memory
//                    (offsets, and padded offsets with each expert's range a
//                    multiple of 128 rows; CTA 0 stores both), then its warps
//                    walk 32-slot steps of their part of the chunk in order;
//                    __match_any_sync gives the rank among equal experts
//                    inside a step, running per-warp counters keep the order
//                    across steps, so the sort is stable.
// ===========================================================================
constexpr int kPermWarps = 8;
constexpr int kPad = 128;
constexpr int kScanWarps = 32;

// A chunk is kPermWarps * slots_per_warp consecutive slots, one CTA each.
int permute_chunks(int64_t slots, int slots_per_warp) {
  const int64_t chunk = static_cast<int64_t>(kPermWarps) * slots_per_warp;
  return static_cast<int>((slots + chunk - 1) / chunk);
}

__global__ void __launch_bounds__(256) perm_count_kernel(const int32_t* __restrict__ idx,
                                                         int64_t slots, int N, int spw, int nch,
                                                         int32_t* __restrict__ cnt, DevErr err) {
  pdl_begin();
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < N; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t chunk = static_cast<int64_t>(kPermWarps) * spw;
  const int64_t f0 = static_cast<int64_t>(blockIdx.x) * chunk;
  const int64_t f1 = min(slots, f0 + chunk);
  for (int64_t f = f0 + threadIdx.x; f < f1; f += blockDim.x) {
    const int e = __ldg(idx + f);
    if (e < 0 || e >= N) {
      dev_report(err, kErrBounds, static_cast<uint32_t>(f));
      continue;
    }
    atomicAdd(&hist[e], 1);   // shared-memory counter; global buffers are written once below
  }
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x) cnt[static_cast<int64_t>(e) * nch + blockIdx.x] = hist[e];
}

// Warp per expert: exclusive prefix of its chunk counts, total at the end.
__global__ void __launch_bounds__(kScanWarps * 32) perm_scan_kernel(int32_t* __restrict__ cnt, int nch, int N) {
  pdl_begin();
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * kScanWarps + (threadIdx.x >> 5);
  if (e >= N) return;
  int32_t* row = cnt + static_cast<int64_t>(e) * nch;
  int carry = 0;
  for (int c0 = 0; c0 < nch; c0 += 32) {
    const int c = c0 + lane;
    const int v = c < nch ? row[c] : 0;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (c < nch) row[c] = carry + x - v;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) cnt[static_cast<int64_t>(N) * nch + e] = carry;
}

// Exclusive scan of v over a 256-thread block; *total gets the block's sum.
__device__ __forceinline__ int block256_exclusive_scan(int v, int* smem_warp, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) smem_warp[wid] = x;
  __syncthreads();
  int base = 0, all = 0;
#pragma unroll
  for (int w2 = 0; w2 < 8; ++w2) {
    const int sw = smem_warp[w2];
    if (w2 < wid) base += sw;
    all += sw;
  }
  __syncthreads();
  *total = all;
  return base + x - v;
}

__global__ void __launch_bounds__(256) perm_scatter_kernel(
    const int32_t* __restrict__ idx, int64_t slots, int N, int spw, int nch, const int32_t* __restrict__ cnt,
    int32_t* __restrict__ offsets_out, int32_t* __restrict__ poff_out,
    int32_t* __restrict__ perm_src, int32_t* __restrict__ inv_perm,
    const float* __restrict__ topk_w, float* __restrict__ perm_gate, int32_t* __restrict__ slot_row) {
  pdl_begin();
  extern __shared__ int32_t sm[];
  int32_t* wcnt = sm;                          // [kPermWarps][N]
  int32_t* s_off = sm + kPermWarps * N;        // [N]
  int32_t* s_poff = s_off + N;                 // [N]
  __shared__ int warp_sums[8];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  // offsets and padded offsets of all experts from their totals: each thread
  // owns four consecutive experts (N <= 1024)
  {
    const int32_t* tot = cnt + static_cast<int64_t>(N) * nch;
    int v[4], pv[4], sum = 0, psum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = threadIdx.x * 4 + i;
      v[i] = e < N ? __ldg(tot + e) : 0;
      pv[i] = ((v[i] + kPad - 1) / kPad) * kPad;
      sum += v[i];
      psum += pv[i];
    }
    int total = 0, ptotal = 0;
    int run = block256_exclusive_scan(sum, warp_sums, &total);
    int prun = block256_exclusive_scan(psum, warp_sums, &ptotal);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = threadIdx.x * 4 + i;
      if (e < N) {
        s_off[e] = run;
        s_poff[e] = prun;
        if (blockIdx.x == 0) {
          offsets_out[e] = run;
          poff_out[e] = prun;
        }
      }
      run += v[i];
      prun += pv[i];
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      offsets_out[N] = total;
      poff_out[N] = ptotal;
    }
  }
  for (int i = threadIdx.x; i < kPermWarps * N; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  const int64_t f0 = (static_cast<int64_t>(blockIdx.x) * kPermWarps + wid) * spw;
  const int64_t f1 = min(slots, f0 + spw);
  int32_t* my = wcnt + wid * N;
  const unsigned lt = (1u << lane) - 1u;
  // per-warp counts
  for (int64_t s = f0; s < f1; s += 32) {
    const int64_t f = s + lane;
    const bool live = f < f1;
    int e = live ? __ldg(idx + f) : -1;
    if (e >= N) e = -1;   // out of range: reported by the count pass, skipped here
    const unsigned act = __ballot_sync(0xffffffffu, live && e >= 0);
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (live && e >= 0 && (peers & act & lt) == 0) my[e] += __popc(peers & act);
    __syncwarp();
  }
  __syncthreads();
  // exclusive prefix over the warps of this chunk, per expert
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    int run = 0;
    for (int w2 = 0; w2 < kPermWarps; ++w2) {
      const int c = wcnt[w2 * N + e];
      wcnt[w2 * N + e] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int64_t s = f0; s < f1; s += 32) {
    const int64_t f = s + lane;
    const bool live = f < f1;
    int e = live ? __ldg(idx + f) : -1;
    if (e >= N) e = -1;
    const unsigned act = __ballot_sync(0xffffffffu, live && e >= 0);
    const unsigned peers = __match_any_sync(0xffffffffu, e) & act;
    int r = 0;
    if (live && e >= 0) {
      r = s_off[e] + __ldg(cnt + static_cast<int64_t>(e) * nch + blockIdx.x) + my[e] + __popc(peers & lt);
    }
    __syncwarp();
    if (live && e >= 0) {
      if ((peers & lt) == 0) my[e] += __popc(peers);
      perm_src[r] = static_cast<int32_t>(f);
      inv_perm[f] = r;
      const int p = r - s_off[e] + s_poff[e];
      if (perm_gate) perm_gate[p] = __ldg(topk_w + f);
      if (slot_row) slot_row[f] = p;
    } else if (live && slot_row) {
      slot_row[f] = -1;   // a slot left out (expert index out of range)
    }
    __syncwarp();
  }
}

lmoe_status launch_permute(const int32_t* idx, int64_t T, int K, int N, int32_t* offsets,
                           int32_t* perm_src, int32_t* inv_perm, int32_t* padded_offsets,
                           int32_t* scratch, const float* topk_w, float* perm_gate,
                           uint32_t* err, cudaStream_t s, int slots_per_warp, int32_t* slot_row) {
  if (N > 1024) return LMOE_ERR_UNSUPPORTED;
  if (slots_per_warp <= 0 || slots_per_warp % 32) return LMOE_ERR_INVALID_ARG;
  const int64_t slots = T * K;
  const int nch = permute_chunks(slots, slots_per_warp);
  DevErr de{err};
  if (nch > 0) {
    launch_k(perm_count_kernel, dim3(nch), dim3(256), N * sizeof(int32_t), s, idx, slots, N, slots_per_warp, nch,
             scratch, de);
    count_launch();
  }
  launch_k(perm_scan_kernel, dim3((N + kScanWarps - 1) / kScanWarps), dim3(kScanWarps * 32), 0, s, scratch, nch, N);
  count_launch();
  // at least one CTA: it also stores the offsets (all zero without slots)
  const size_t sm = (static_cast<size_t>(kPermWarps) + 2) * N * sizeof(int32_t);
  launch_k(perm_scatter_kernel, dim3(nch > 0 ? nch : 1), dim3(256), sm, s, idx, slots, N, slots_per_warp, nch,
           static_cast<const int32_t*>(scratch), offsets, padded_offsets, perm_src, inv_perm, topk_w, perm_gate,
           slot_row);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

// ===========================================================================
// Gather token rows into the padded expert-grouped buffer: one warp per
// sorted position, 16-byte loads and stores. NVFP4 block scales move from the
// row-major [T][cols/16] layout to the MMA-tiled layout at the padded row.
// ===========================================================================
__device__ __forceinline__ int64_t sf_tiled_offset(int64_t row, int j, int groups64) {
  const int64_t atom = (row >> 7) * groups64 + (j >> 2);
  return atom * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (j & 3);
}

__global__ void __launch_bounds__(256) gather_kernel(
    const int32_t* __restrict__ idx, const int32_t* __restrict__ perm_src,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ poff, int64_t slots, int K, int N,
    const uint8_t* __restrict__ rows, int64_t row_bytes, uint8_t* __restrict__ out,
    const uint8_t* __restrict__ rows_sf, uint8_t* __restrict__ out_sf) {
  pdl_begin();
  const int lane = threadIdx.x & 31;
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  // sorted positions past offsets[N] exist only when some expert index was out
  // of range (the permutation leaves those slots out): nothing to copy there
  if (r >= slots || r >= __ldg(offsets + N)) return;
  const int f = __ldg(perm_src + r);
  const int t = f / K;
  const int e = __ldg(idx + f);
  const int64_t p = r - __ldg(offsets + e) + __ldg(poff + e);
  if (out) {
    const uint4* src = reinterpret_cast<const uint4*>(rows + static_cast<int64_t>(t) * row_bytes);
    uint4* dst = reinterpret_cast<uint4*>(out + p * row_bytes);
    const int64_t n16 = row_bytes >> 4;
    // the permuted copy streams through L2 (evict first) so the source rows,
    // read K times, stay
    const uint64_t pol = policy_evict_first();
    int64_t i = lane;
    for (; i + 96 < n16; i += 128) {   // four 16-byte loads in flight per lane
      const uint4 v0 = __ldg(src + i), v1 = __ldg(src + i + 32), v2 = __ldg(src + i + 64), v3 = __ldg(src + i + 96);
      st_global_v4_hint(dst + i, v0, pol);
      st_global_v4_hint(dst + i + 32, v1, pol);
      st_global_v4_hint(dst + i + 64, v2, pol);
      st_global_v4_hint(dst + i + 96, v3, pol);
    }
    for (; i < n16; i += 32) st_global_v4_hint(dst + i, __ldg(src + i), pol);
  }
  if (out_sf) {
    const int cols = static_cast<int>(row_bytes * 2);
    const int nsf = cols / 16;
    const int groups64 = (cols + 63) / 64;
    const uint8_t* src = rows_sf + static_cast<int64_t>(t) * nsf;
    for (int j = lane * 4; j < nsf; j += 128) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        if (j + b < nsf) word |= static_cast<uint32_t>(__ldg(src + j + b)) << (8 * b);
      *reinterpret_cast<uint32_t*>(out_sf + sf_tiled_offset(p, j, groups64)) = word;
    }
  }
}

lmoe_status launch_gather(const int32_t* idx, const int32_t* perm_src, const int32_t* offsets,
                          const int32_t* padded_offsets, int64_t slots, int K, const void* rows,
                          int64_t row_bytes, void* out_rows, const uint8_t* rows_sf,
                          uint8_t* out_sf, int N, cudaStream_t s) {
  if (slots == 0) return LMOE_OK;
  const int64_t blocks = (slots * 32 + 255) / 256;
  launch_k(gather_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, idx, perm_src, offsets,
           padded_offsets, slots, K, N, static_cast<const uint8_t*>(rows), row_bytes, static_cast<uint8_t*>(out_rows),
           rows_sf, out_sf);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

// ===========================================================================
// Combine: c_t = sum_k w_tk * y[row(t,k)], fp32 in k order, one CTA per token.
// ===========================================================================
template <typename TA>
__global__ void __launch_bounds__(256) combine_kernel(
    const TA* __restrict__ y, const int32_t* __restrict__ idx, const int32_t* __restrict__ inv_perm,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ poff, const float* __restrict__ w,
    const TA* __restrict__ resid, TA* __restrict__ c, int K, int N, int l) {
  pdl_begin();
  extern __shared__ int64_t rowk[];   // [K] padded rows of the token's in-range slots, in k order
  __shared__ float wk[32];
  __shared__ int s_nk;
  const int64_t t = blockIdx.x;
  if (threadIdx.x < 32) {
    // an out-of-range expert index contributes nothing (the permutation left
    // its slot out and reported it); the others keep their k order
    const int k = threadIdx.x;
    bool ok = false;
    int64_t row = 0;
    float g = 0.0f;
    if (k < K) {
      const int64_t f = t * K + k;
      const int e = __ldg(idx + f);
      ok = e >= 0 && e < N;
      if (ok) {
        row = static_cast<int64_t>(__ldg(inv_perm + f)) - __ldg(offsets + e) + __ldg(poff + e);
        g = w ? __ldg(w + f) : 1.0f;
        // debug build: a row outside the padded rows (caller-supplied offsets) is skipped
        if (kChecks && (row < 0 || row >= __ldg(poff + N))) ok = false;
      }
    }
    const unsigned m = __ballot_sync(0xffffffffu, ok);
    if (ok) {
      const int pos = __popc(m & ((1u << k) - 1u));
      rowk[pos] = row;
      wk[pos] = g;
    }
    if (k == 0) s_nk = __popc(m);
  }
  __syncthreads();
  const int nk = s_nk;
  constexpr int V = 16 / sizeof(TA);   // elements per 16-byte vector
  for (int col = threadIdx.x * V; col < l; col += blockDim.x * V) {
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.0f;
    auto add = [&](const uint4& u, float g) {
      if constexpr (sizeof(TA) == 2) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f2 = __bfloat1622float2(h[i]);
          acc[2 * i] += g * f2.x;
          acc[2 * i + 1] += g * f2.y;
        }
      } else {
        const float* f4 = reinterpret_cast<const float*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += g * f4[i];
      }
    };
    // four of the token's rows in flight at a time; the sums stay in k order
    int k = 0;
    for (; k + 4 <= nk; k += 4) {
      uint4 u[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) u[q] = __ldg(reinterpret_cast<const uint4*>(y + rowk[k + q] * l + col));
#pragma unroll
      for (int q = 0; q < 4; ++q) add(u[q], wk[k + q]);
    }
    for (; k < nk; ++k) add(__ldg(reinterpret_cast<const uint4*>(y + rowk[k] * l + col)), wk[k]);
    if (resid) {   // + a [T, l] term (the shared experts' output) after the K routed rows
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(resid + t * l + col));
      if constexpr (sizeof(TA) == 2) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f2 = __bfloat1622float2(h[i]);
          acc[2 * i] += f2.x;
          acc[2 * i + 1] += f2.y;
        }
      } else {
        const float* f4 = reinterpret_cast<const float*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += f4[i];
      }
    }
    uint4 o;
    if constexpr (sizeof(TA) == 2) {
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
    } else {
      o.x = __float_as_uint(acc[0]);
      o.y = __float_as_uint(acc[1]);
      o.z = __float_as_uint(acc[2]);
      o.w = __float_as_uint(acc[3]);
    }
    *reinterpret_cast<uint4*>(c + t * l + col) = o;
  }
}

lmoe_status launch_combine(const void* y, int act, const int32_t* idx, const int32_t* inv_perm,
                           const int32_t* offsets, const int32_t* padded_offsets, const float* w,
                           const void* resid, void* c, int64_t T, int K, int N, int l, cudaStream_t s) {
  if (T == 0) return LMOE_OK;
  if (K > 32) return LMOE_ERR_UNSUPPORTED;
  const size_t sm = static_cast<size_t>(K) * sizeof(int64_t);
  if (act == LMOE_BF16)
    launch_k(combine_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(T)), dim3(256), sm, s,
             static_cast<const __nv_bfloat16*>(y), idx, inv_perm, offsets, padded_offsets, w,
             static_cast<const __nv_bfloat16*>(resid), static_cast<__nv_bfloat16*>(c), K, N, l);
  else
    launch_k(combine_kernel<float>, dim3(static_cast<unsigned>(T)), dim3(256), sm, s, static_cast<const float*>(y),
             idx, inv_perm, offsets, padded_offsets, w, static_cast<const float*>(resid), static_cast<float*>(c), K,
             N, l);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

// ===========================================================================
// NVFP4 quantiser.
//   pass 1: |x| max with one partial per CTA (no float atomics).
//   pass 2: every CTA reduces the partials (same order -> same s_g), then one
//           thread per 16-element block: E4M3 block scale and E2M1 codes with
//           the hardware round-to-nearest-even, satfinite conversions.
// ===========================================================================
constexpr int kQThreads = 256;

int nvfp4_partials(int64_t elems) {
  const int64_t want = (elems + 8 * 1024 - 1) / (8 * 1024);
  return static_cast<int>(want < 1 ? 1 : (want > 1184 ? 1184 : want));
}

template <typename TI>
__device__ __forceinline__ float load_abs_max(const TI* p, int64_t i) {
  return fabsf(static_cast<float>(p[i]));
}

template <typename TI>
__global__ void __launch_bounds__(kQThreads) nvfp4_amax_kernel(const TI* __restrict__ in, int64_t n,
                                                               float* __restrict__ partials) {
  pdl_begin();
  __shared__ float red[kQThreads / 32];
  float m = 0.0f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    m = fmaxf(m, fabsf(static_cast<float>(in[i])));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = 0.0f;
    for (int i = 0; i < kQThreads / 32; ++i) r = fmaxf(r, red[i]);
    partials[blockIdx.x] = r;
  }
}

// E4M3 code -> value (exact): subnormal f * 2^-9, normal (8 + f) * 2^(e - 10).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const int e = (c >> 3) & 15, f = c & 7;
  return e == 0 ? ldexpf(static_cast<float>(f), -9) : ldexpf(static_cast<float>(8 + f), e - 10);
}

// fp32 -> E4M3 (round to nearest even, saturating to 448): PTX cvt.
__device__ __forceinline__ uint32_t cvt_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

// Every CTA reduces the per-CTA maxima the same way (max is exact, so the
// order does not matter) and derives s_g = fp32(amax / divisor), 1 when amax
// = 0 (divisor 2688 = 6 * 448 for NVFP4, 448 for FP8).
__device__ __forceinline__ float cta_global_scale(const float* partials, int np, const float* global_in,
                                                  float divisor = 2688.0f) {
  __shared__ float red[kQThreads / 32];
  __shared__ float result;
  if (global_in) return __ldg(global_in);
  float m = 0.0f;
  for (int i = threadIdx.x; i < np; i += blockDim.x) m = fmaxf(m, __ldg(partials + i));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = 0.0f;
    for (int i = 0; i < kQThreads / 32; ++i) r = fmaxf(r, red[i]);
    result = r == 0.0f ? 1.0f : __fdiv_rn(r, divisor);
  }
  __syncthreads();
  return result;
}

template <typename TI>
__device__ __forceinline__ void load16(const TI* src, float (&x)[16]) {
  if constexpr (sizeof(TI) == 2) {
    const uint4* p = reinterpret_cast<const uint4*>(src);
    const uint4 u0 = __ldg(p), u1 = __ldg(p + 1);
    const __nv_bfloat162* h0 = reinterpret_cast<const __nv_bfloat162*>(&u0);
    const __nv_bfloat162* h1 = reinterpret_cast<const __nv_bfloat162*>(&u1);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 a = __bfloat1622float2(h0[i]);
      const float2 b = __bfloat1622float2(h1[i]);
      x[2 * i] = a.x;
      x[2 * i + 1] = a.y;
      x[8 + 2 * i] = b.x;
      x[8 + 2 * i + 1] = b.y;
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(src);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldg(p + i);
      x[4 * i] = v.x;
      x[4 * i + 1] = v.y;
      x[4 * i + 2] = v.z;
      x[4 * i + 3] = v.w;
    }
  }
}

// Quantise one 16-element block: returns the E4M3 scale code, writes 8 code bytes.
__device__ __forceinline__ uint32_t nvfp4_block(const float (&x)[16], float s_g, uint2& codes) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const float t = __fmul_rn(s_g, 6.0f);
  const uint32_t sb = cvt_e4m3(__fdiv_rn(amax, t));
  const float dec = e4m3_value(sb);
  uint32_t lo = 0, hi = 0;
  if (dec != 0.0f) {
    const float sc = __fmul_rn(dec, s_g);
    const uint2 c = e2m1_codes16(x, sc, __frcp_rn(sc));   // codes of RN(x / sc)
    lo = c.x;
    hi = c.y;
  }
  codes.x = lo;
  codes.y = hi;
  return sb;
}

template <typename TI>
__global__ void __launch_bounds__(kQThreads) nvfp4_encode_kernel(
    const TI* __restrict__ in, int64_t rows, int64_t cols, const float* __restrict__ partials, int np,
    const float* __restrict__ global_in, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
    float* __restrict__ global_out, int tiled) {
  pdl_begin();
  const float s_g = cta_global_scale(partials, np, global_in);
  if (blockIdx.x == 0 && threadIdx.x == 0 && global_out) *global_out = s_g;
  const int64_t nb = cols / 16;
  // tiled layout: cover the padded grid so that padding scale bytes are zero
  const int64_t rows_cov = tiled ? ((rows + 127) / 128) * 128 : rows;
  const int64_t nb_cov = tiled ? ((cols + 63) / 64) * 4 : nb;
  const int groups64 = static_cast<int>((cols + 63) / 64);
  const int64_t total = rows_cov * nb_cov;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < total;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = b / nb_cov, j = b % nb_cov;
    uint32_t scode = 0;
    if (r < rows && j < nb) {
      float x[16];
      load16<TI>(in + r * cols + j * 16, x);
      uint2 c;
      scode = nvfp4_block(x, s_g, c);
      *reinterpret_cast<uint2*>(codes + r * (cols / 2) + j * 8) = c;
    }
    if (tiled) sf[sf_tiled_offset(r, static_cast<int>(j), groups64)] = static_cast<uint8_t>(scode);
    else sf[r * nb + j] = static_cast<uint8_t>(scode);
  }
}

// Two-dimensional blocks: one thread per 16-row group x 16-column block. The
// scale comes from the amax over the block's (up to) 256 elements; each of its
// rows is then quantised with it and carries it in its own scale entry, so
// the output has the 1 x 16 layout and every consumer reads it unchanged.
template <typename TI>
__global__ void __launch_bounds__(kQThreads) nvfp4_encode2d_kernel(
    const TI* __restrict__ in, int64_t rows, int64_t cols, const float* __restrict__ partials, int np,
    const float* __restrict__ global_in, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
    float* __restrict__ global_out, int tiled) {
  pdl_begin();
  const float s_g = cta_global_scale(partials, np, global_in);
  if (blockIdx.x == 0 && threadIdx.x == 0 && global_out) *global_out = s_g;
  const int64_t nb = cols / 16;
  const int64_t rows_cov = tiled ? ((rows + 127) / 128) * 128 : rows;
  const int64_t nb_cov = tiled ? ((cols + 63) / 64) * 4 : nb;
  const int groups64 = static_cast<int>((cols + 63) / 64);
  const int64_t total = ((rows_cov + 15) / 16) * nb_cov;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < total;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r0 = (b / nb_cov) * 16, j = b % nb_cov;
    const int64_t r1 = r0 + 16 < rows_cov ? r0 + 16 : rows_cov;
    const int nr = (j < nb && r0 < rows) ? static_cast<int>(rows - r0 < 16 ? rows - r0 : 16) : 0;
    uint32_t scode = 0;
    if (nr > 0) {
      float x[16];
      float amax = 0.0f;
      for (int i = 0; i < nr; ++i) {
        load16<TI>(in + (r0 + i) * cols + j * 16, x);
#pragma unroll
        for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(x[e]));
      }
      scode = cvt_e4m3(__fdiv_rn(amax, __fmul_rn(s_g, 6.0f)));
      const float dec = e4m3_value(scode);
      const float sc = __fmul_rn(dec, s_g);
      const float rc = dec != 0.0f ? __frcp_rn(sc) : 0.0f;
      for (int i = 0; i < nr; ++i) {
        uint2 c = make_uint2(0u, 0u);
        if (dec != 0.0f) {
          load16<TI>(in + (r0 + i) * cols + j * 16, x);
          c = e2m1_codes16(x, sc, rc);   // codes of RN(x / sc)
        }
        *reinterpret_cast<uint2*>(codes + (r0 + i) * (cols / 2) + j * 8) = c;
      }
    }
    for (int64_t r = r0; r < r1; ++r) {
      const uint8_t v = (r < rows && j < nb) ? static_cast<uint8_t>(scode) : 0;
      if (tiled) sf[sf_tiled_offset(r, static_cast<int>(j), groups64)] = v;
      else sf[r * nb + j] = v;
    }
  }
}

// NVFP4 codes of each token row written straight to the padded rows of its K
// slots (the permutation's slot_row; -1 marks a slot left out), with the
// block scales in the MMA-tiled layout at those rows: the quantiser and the
// dispatch gather in one pass, so the row-major codes are never stored. A
// warp per token; each lane quantises 64 consecutive elements (four blocks)
// and stores their 32 code bytes and 4 scale bytes at every slot row.
template <typename TI>
__global__ void __launch_bounds__(kQThreads) nvfp4_encode_scatter_kernel(
    const TI* __restrict__ in, int64_t rows, int cols, const float* __restrict__ partials, int np,
    const int32_t* __restrict__ slot_row, int K, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
    float* __restrict__ global_out) {
  pdl_begin();
  const float s_g = cta_global_scale(partials, np, nullptr);
  if (blockIdx.x == 0 && threadIdx.x == 0 && global_out) *global_out = s_g;
  constexpr unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int groups64 = cols / 64;
  const int64_t row_bytes = cols / 2;
  const uint64_t pol = policy_evict_first();   // the expert GEMM reads the slot rows much later
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; t < rows; t += warps) {
    const int my_row = lane < K ? __ldg(slot_row + t * K + lane) : -1;
    for (int g0 = 0; g0 < groups64; g0 += 32) {
      const int g = g0 + lane;
      uint4 c01 = make_uint4(0u, 0u, 0u, 0u), c23 = c01;
      uint32_t sw = 0;
      if (g < groups64) {
        const TI* src = in + t * cols + static_cast<int64_t>(g) * 64;
        float x[16];
        uint2 c;
        load16<TI>(src, x);
        sw = nvfp4_block(x, s_g, c);
        c01.x = c.x;
        c01.y = c.y;
        load16<TI>(src + 16, x);
        sw |= nvfp4_block(x, s_g, c) << 8;
        c01.z = c.x;
        c01.w = c.y;
        load16<TI>(src + 32, x);
        sw |= nvfp4_block(x, s_g, c) << 16;
        c23.x = c.x;
        c23.y = c.y;
        load16<TI>(src + 48, x);
        sw |= nvfp4_block(x, s_g, c) << 24;
        c23.z = c.x;
        c23.w = c.y;
      }
      for (int k = 0; k < K; ++k) {
        const int p = __shfl_sync(FULL, my_row, k);
        if (p < 0 || g >= groups64) continue;
        uint8_t* dst = codes + static_cast<int64_t>(p) * row_bytes + static_cast<int64_t>(g) * 32;
        // the lane's 32 code bytes as one 32-byte store: whole sectors, half the requests
        const uint32_t u[8] = {c01.x, c01.y, c01.z, c01.w, c23.x, c23.y, c23.z, c23.w};
        st_global_v8_hint(dst, u, pol);
        *reinterpret_cast<uint32_t*>(sf + sf_tiled_offset(p, g * 4, groups64)) = sw;
      }
    }
  }
}

lmoe_status launch_nvfp4_quantize_scatter(const void* in, int64_t rows, int cols, const int32_t* slot_row, int K,
                                          uint8_t* codes, uint8_t* sf, float* global_out, float* partials,
                                          int npartials, cudaStream_t s) {
  if (rows == 0) return LMOE_OK;
  if (cols % 64 || K < 1 || K > 32) return LMOE_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(codes) & 31) return LMOE_ERR_INVALID_ARG;   // 32-byte code stores
  launch_k(nvfp4_amax_kernel<__nv_bfloat16>, dim3(npartials), dim3(kQThreads), 0, s,
           static_cast<const __nv_bfloat16*>(in), rows * cols, partials);
  count_launch();
  const int sms = device_sm_count();
  int64_t blocks = (rows * 32 + kQThreads - 1) / kQThreads;
  if (blocks > static_cast<int64_t>(sms) * 8) blocks = static_cast<int64_t>(sms) * 8;
  launch_k(nvfp4_encode_scatter_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(blocks)), dim3(kQThreads), 0, s,
           static_cast<const __nv_bfloat16*>(in), rows, cols, static_cast<const float*>(partials), npartials,
           slot_row, K, codes, sf, global_out);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

// Dispatch copy in token order: each token's row is read once and written to
// the padded rows of its K slots (the permutation's slot_row; -1 marks a slot
// left out). A warp per token; each pass holds 2 KB of the row in registers
// (four 16-byte loads per lane) and stores it at every slot row.
__global__ void __launch_bounds__(256) scatter_rows_kernel(const uint8_t* __restrict__ rows, int64_t n,
                                                           int64_t row_bytes, const int32_t* __restrict__ slot_row,
                                                           int K, uint8_t* __restrict__ out) {
  pdl_begin();
  constexpr unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int64_t n16 = row_bytes >> 4;
  const uint64_t pol = policy_evict_first();   // the expert GEMM reads the slot rows much later
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; t < n; t += warps) {
    const int my_row = lane < K ? __ldg(slot_row + t * K + lane) : -1;
    const uint4* src = reinterpret_cast<const uint4*>(rows + t * row_bytes);
    for (int64_t i0 = 0; i0 < n16; i0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i = i0 + u * 32 + lane;
        v[u] = i < n16 ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
      }
      for (int k = 0; k < K; ++k) {
        const int p = __shfl_sync(FULL, my_row, k);
        if (p < 0) continue;
        uint4* dst = reinterpret_cast<uint4*>(out + static_cast<int64_t>(p) * row_bytes);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t i = i0 + u * 32 + lane;
          if (i < n16) st_global_v4_hint(dst + i, v[u], pol);
        }
      }
    }
  }
}

lmoe_status launch_scatter_rows(const void* rows, int64_t n, int64_t row_bytes, const int32_t* slot_row, int K,
                                void* out, cudaStream_t s) {
  if (n == 0) return LMOE_OK;
  if (row_bytes <= 0 || row_bytes % 16 || K < 1 || K > 32) return LMOE_ERR_UNSUPPORTED;
  const int sms = device_sm_count();
  int64_t blocks = (n * 32 + 255) / 256;
  if (blocks > static_cast<int64_t>(sms) * 8) blocks = static_cast<int64_t>(sms) * 8;
  launch_k(scatter_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
           static_cast<const uint8_t*>(rows), n, row_bytes, slot_row, K, static_cast<uint8_t*>(out));
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

lmoe_status launch_nvfp4_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols,
                                  const float* global_in, uint8_t* codes, uint8_t* sf,
                                  float* global_out, int sf_layout, float* partials, int npartials,
                                  uint32_t* err, cudaStream_t s) {
  (void)err;
  const int64_t n = rows * cols;
  if (!global_in) {
    if (in_dtype == LMOE_BF16)
      launch_k(nvfp4_amax_kernel<__nv_bfloat16>, dim3(npartials), dim3(kQThreads), 0, s,
               static_cast<const __nv_bfloat16*>(in), n, partials);
    else
      launch_k(nvfp4_amax_kernel<float>, dim3(npartials), dim3(kQThreads), 0, s, static_cast<const float*>(in), n,
               partials);
    count_launch();
  }
  const bool blk2d = (sf_layout & LMOE_SF_BLOCK_16X16) != 0;
  const int tiled = (sf_layout & ~LMOE_SF_BLOCK_16X16) == LMOE_SF_MMA_TILED;
  const int64_t rows_cov = tiled ? ((rows + 127) / 128) * 128 : rows;
  const int64_t nb_cov = tiled ? ((cols + 63) / 64) * 4 : cols / 16;
  const int64_t total = (blk2d ? (rows_cov + 15) / 16 : rows_cov) * nb_cov;
  const int sms = device_sm_count();
  int64_t blocks = (total + kQThreads - 1) / kQThreads;
  if (blocks > static_cast<int64_t>(sms) * 8) blocks = static_cast<int64_t>(sms) * 8;
  if (blocks < 1) blocks = 1;
  if (blk2d) {
    if (in_dtype == LMOE_BF16)
      launch_k(nvfp4_encode2d_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(blocks)), dim3(kQThreads), 0, s,
               static_cast<const __nv_bfloat16*>(in), rows, cols, static_cast<const float*>(partials),
               global_in ? 0 : npartials, global_in, codes, sf, global_out, tiled);
    else
      launch_k(nvfp4_encode2d_kernel<float>, dim3(static_cast<unsigned>(blocks)), dim3(kQThreads), 0, s,
               static_cast<const float*>(in), rows, cols, static_cast<const float*>(partials),
               global_in ? 0 : npartials, global_in, codes, sf, global_out, tiled);
  } else if (in_dtype == LMOE_BF16)
    launch_k(nvfp4_encode_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(blocks)), dim3(kQThreads), 0, s,
             static_cast<const __nv_bfloat16*>(in), rows, cols, static_cast<const float*>(partials),
             global_in ? 0 : npartials, global_in, codes, sf, global_out, tiled);
  else
    launch_k(nvfp4_encode_kernel<float>, dim3(static_cast<unsigned>(blocks)), dim3(kQThreads), 0, s,
             static_cast<const float*>(in), rows, cols, static_cast<const float*>(partials), global_in ? 0 : npartials,
             global_in, codes, sf, global_out, tiled);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

// ===========================================================================
// FP8 (E4M3) with one FP32 scale per tensor (the shared experts' weights and
// activations): s = scale_in ? *scale_in : fp32(amax / 448) (1 when amax = 0);
// q = E4M3_rn_satfinite(fp32(x / s)), the division an IEEE fp32 division as
// the definition states. A thread per 16 elements, 16 code bytes per store.
// ===========================================================================
template <typename TI>
__global__ void __launch_bounds__(kQThreads) fp8_encode_kernel(const TI* __restrict__ in, int64_t n,
                                                               const float* __restrict__ partials, int np,
                                                               const float* __restrict__ scale_in,
                                                               uint8_t* __restrict__ codes,
                                                               float* __restrict__ scale_out) {
  pdl_begin();
  const float s = cta_global_scale(partials, np, scale_in, 448.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0 && scale_out) *scale_out = s;
  const int64_t nv = n / 16;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < nv;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float x[16];
    load16<TI>(in + v * 16, x);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      w[j] = cvt_e4m3(__fdiv_rn(x[4 * j], s)) | (cvt_e4m3(__fdiv_rn(x[4 * j + 1], s)) << 8) |
             (cvt_e4m3(__fdiv_rn(x[4 * j + 2], s)) << 16) | (cvt_e4m3(__fdiv_rn(x[4 * j + 3], s)) << 24);
    *reinterpret_cast<uint4*>(codes + v * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

lmoe_status launch_fp8_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols, const float* scale_in,
                                uint8_t* codes, float* scale_out, float* partials, int npartials, cudaStream_t s) {
  const int64_t n = rows * cols;
  if (n == 0) return LMOE_OK;
  if (!scale_in) {
    if (in_dtype == LMOE_BF16)
      launch_k(nvfp4_amax_kernel<__nv_bfloat16>, dim3(npartials), dim3(kQThreads), 0, s,
               static_cast<const __nv_bfloat16*>(in), n, partials);
    else
      launch_k(nvfp4_amax_kernel<float>, dim3(npartials), dim3(kQThreads), 0, s, static_cast<const float*>(in), n,
               partials);
    count_launch();
  }
  const int sms = device_sm_count();
  int64_t blocks = (n / 16 + kQThreads - 1) / kQThreads;
  if (blocks > static_cast<int64_t>(sms) * 8) blocks = static_cast<int64_t>(sms) * 8;
  if (blocks < 1) blocks = 1;
  const int np = scale_in ? 0 : npartials;
  if (in_dtype == LMOE_BF16)
    launch_k(fp8_encode_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(blocks)), dim3(kQThreads), 0, s,
             static_cast<const __nv_bfloat16*>(in), n, static_cast<const float*>(partials), np, scale_in, codes,
             scale_out);
  else
    launch_k(fp8_encode_kernel<float>, dim3(static_cast<unsigned>(blocks)), dim3(kQThreads), 0, s,
             static_cast<const float*>(in), n, static_cast<const float*>(partials), np, scale_in, codes, scale_out);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

// ===========================================================================
// Failure-path self test: one thread waits on an mbarrier nothing arrives
// on, through the pipelines' bounded wait with a short limit; the wait gives
// up, records a timeout (info 0x7001) in the error word and the kernel
// returns, leaving the context usable.
// ===========================================================================
__global__ void __launch_bounds__(32) selftest_wait_kernel(DevErr err, long long limit) {
  pdl_begin();
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, err, 0x7001, limit);
}

lmoe_status launch_selftest_wait(uint32_t* err, long long limit, cudaStream_t s) {
  launch_k(selftest_wait_kernel, dim3(1), dim3(32), 0, s, DevErr{err}, limit);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

}  // namespace lmoe
