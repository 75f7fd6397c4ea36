// Grouped BF16 expert GEMM on CTA pairs (tcgen05 cta_group::2), weight-major:
//
//   D[w, t] = sum_k W_e[w, k] . X[t, k]     w: 256 output features of expert e
//                                            t: up to 256 of the expert's tokens
//
// Two CTAs of a cluster share one 256 x N tile: CTA r loads weight rows
// w0 + 128 r .. + 127 (A) and its half of the token rows (B, N/2 rows), the
// even CTA issues tcgen05.mma.cta_group::2 (M = 256) that reads both CTAs'
// shared memory, and each CTA's tensor memory receives the accumulator rows
// of its own 128 features. Per CTA and K block this moves 16 KB of weights
// and at most 16 KB of tokens for the work a single-CTA 128 x 256 tile does
// with 48 KB, so six stages fit where four did.
//
// Synchronisation (all waits bounded):
//   full[s]    even CTA only: its producer arms it with both CTAs' bytes; the
//              loads of both CTAs complete on it (cta_group::2 TMA).
//   empty[s]   both CTAs: the MMA's commit is multicast to the pair.
//   tfull[a]   both CTAs: accumulator a ready (multicast commit).
//   tempty[a]  even CTA: eight arrivals, four epilogue warps per CTA.
// The pair allocates and frees its TMEM together, and a cluster barrier
// separates set-up and teardown from the pipeline.
// No TMA load here uses cluster multicast.
#pragma once

#include "gemm_tc.cuh"

namespace lmoe {

__device__ __forceinline__ uint32_t cluster_cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
  return out;
}

__device__ __forceinline__ void cluster_barrier() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA tile load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (cluster address).
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at this shared offset in every CTA of `mask`
// when the pair's tcgen05 operations issued so far have completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

struct Tc2Smem {
  static constexpr int kABytes = 128 * 128;   // 128 weight rows x 64 bf16 (one K atom)
  static constexpr int kBBytes = 128 * 128;   // up to 128 token rows x 64 bf16
  static constexpr int kAtoms = 2;            // 64-wide K atoms per stage (measured 9% faster than 1)
  static constexpr int kStageBytes = kAtoms * (kABytes + kBBytes);   // A atoms, then B atoms
  static constexpr int kStages = 6 / kAtoms;
  static constexpr int kBarOffset = kStages * kStageBytes;
  // full[S], empty[S], tfull[2], tempty[2], drain, tmem ptr, abort
  static constexpr int kPrefixOffset = kBarOffset + (2 * kStages + 5) * 8 + 16;
  static constexpr int kMaxGroups = 1024;
  static constexpr int kEpiOffset = (kPrefixOffset + (kMaxGroups + 1) * 4 + 15) / 16 * 16;
  // per expert: its row count and first padded row, copied from global memory
  // once, so that no role waits on a global load at a tile boundary
  static constexpr int kExpertOffset = kEpiOffset + 4 * 32 * 32 * 2;
  static constexpr int kBytes = kExpertOffset + 2 * kMaxGroups * 4 + 1024;   // +1024 alignment slack
  static constexpr int kTmemCols = 512;       // two 256-column accumulators
  static constexpr int kTokens = 256;         // tokens per tile (MMA N <= 256)
};

// Pair tile t: expert e, token tile tt (256 tokens), weight tile of 256
// features; the weight tiles of one token tile are consecutive. With a dense
// extra problem its tiles are spread evenly among the grouped ones (tile i is
// an extra tile when floor((i+1) Tx / n) > floor(i Tx / n)), so that its
// tensor work overlaps the weight streaming of the grouped tiles.
struct Tile2 {
  int valid;
  int extra;   // 1: a tile of the dense extra problem
  int expert;
  int act0;    // first token row of the tile (padded grouped row, or row of X)
  int act_n;   // tokens in the tile
  int w0;      // first feature of the pair's 256
  int n;       // MMA N: act_n rounded up to 32
  int kblocks;
};

__device__ __forceinline__ int tc2_extra_tiles(const TcParams& p) {
  return p.rows_x > 0 ? ((p.rows_x + 255) / 256) * ((p.cols_x + 255) / 256) : 0;
}

__device__ __forceinline__ Tile2 tc2_tile(const TcParams& p, int i, int ntiles, int nextra, const int* prefix,
                                          const int* ecount, const int* epoff) {
  Tile2 ti;
  const long long before = static_cast<long long>(i) * nextra / ntiles;
  if (nextra > 0 && static_cast<long long>(i + 1) * nextra / ntiles > before) {
    const int j = static_cast<int>(before);
    const int ntw = (p.cols_x + 255) / 256;
    ti.extra = 1;
    ti.expert = 0;
    ti.w0 = (j % ntw) * 256;
    ti.act0 = (j / ntw) * Tc2Smem::kTokens;
    ti.act_n = min(Tc2Smem::kTokens, p.rows_x - ti.act0);
    ti.valid = ti.act_n > 0;
    ti.n = (ti.act_n + 31) & ~31;
    ti.kblocks = p.kblocks_x;
    return ti;
  }
  const int t = i - static_cast<int>(before);
  ti.extra = 0;
  ti.kblocks = p.seg[0].kblocks;
  const int ntw = (p.cols + 255) / 256;
  int lo = 0, hi = p.groups - 1;   // largest e with prefix[e] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const int e = lo;
  const int n_e = ecount[e];
  const int local = t - prefix[e];
  const int tt = local / ntw, mw = local % ntw;
  ti.expert = e;
  ti.w0 = mw * 256;
  ti.act0 = epoff[e] + tt * Tc2Smem::kTokens;
  ti.act_n = min(Tc2Smem::kTokens, n_e - tt * Tc2Smem::kTokens);
  ti.valid = ti.act_n > 0;
  ti.n = (ti.act_n + 31) & ~31;
  return ti;
}

// Tensor maps: [0] grouped weights (128-row boxes), [1..4] grouped token rows
// with boxes of 128, 64, 32, 16 rows; [5..9] the same for the extra problem.
struct Tc2Maps {
  CUtensorMap m[10];
};

template <int EPI>
__global__ void __launch_bounds__(192, 1)
    tc2_gemm_kernel(const __grid_constant__ Tc2Maps maps, const TcParams p) {
  pdl_begin();
  using S = Tc2Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOffset);
  uint64_t* empty = full + S::kStages;
  uint64_t* tfull = empty + S::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_ptr + 1);
  int* prefix = reinterpret_cast<int*>(smem + S::kPrefixOffset);
  __nv_bfloat16* epi_tile = reinterpret_cast<__nv_bfloat16*>(smem + S::kEpiOffset);
  int* ecount = reinterpret_cast<int*>(smem + S::kExpertOffset);
  int* epoff = ecount + S::kMaxGroups;

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t rank = cluster_cta_rank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;

  // per-expert tile counts -> prefix (every CTA builds its own copy)
  {
    const int ntw = (p.cols + 255) / 256;
    for (int e = threadIdx.x; e < p.groups; e += blockDim.x) {
      int n_e = __ldg(p.offsets + e + 1) - __ldg(p.offsets + e);
      if (kChecks) {   // the expert's rows must fit its padded range inside the buffer
        const int ps = __ldg(p.padded_offsets + e), pe = __ldg(p.padded_offsets + e + 1);
        if (n_e < 0 || ps < 0 || pe > p.rows || ps + n_e > pe) {
          dev_report(p.err, kErrBounds, 0x5200);
          n_e = 0;
        }
      }
      prefix[e + 1] = ((n_e + S::kTokens - 1) / S::kTokens) * ntw;
      ecount[e] = n_e;
      epoff[e] = __ldg(p.padded_offsets + e);
    }
    if (threadIdx.x == 0) prefix[0] = 0;
    __syncthreads();
    if (threadIdx.x < 32) {
      int carry = 0;
      for (int base = 1; base <= p.groups; base += 32) {
        const int i = base + lane;
        int v = i <= p.groups ? prefix[i] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, v, off);
          if (lane >= off) v += y;
        }
        if (i <= p.groups) prefix[i] = v + carry;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
    }
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&maps.m[0]);
    tma_prefetch_desc(&maps.m[1]);
    if (p.rows_x > 0) {
      tma_prefetch_desc(&maps.m[5]);
      tma_prefetch_desc(&maps.m[6]);
    }
  }
  if (warp == 1) tmem_alloc_pair(tmem_ptr, S::kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_barrier();   // both CTAs' barriers and TMEM exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_ptr;
  const int nextra = tc2_extra_tiles(p);
  const int ntiles = prefix[p.groups] + nextra;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      const uint64_t pol_norm = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int t = cluster; t < ntiles && ok; t += nclusters) {
        const Tile2 ti = tc2_tile(p, t, ntiles, nextra, prefix, ecount, epoff);
        if (!ti.valid) continue;
        const int half = ti.n >> 1;
        const int b_row0 = ti.act0 + static_cast<int>(rank) * half;
        const CUtensorMap* amap = &maps.m[ti.extra ? 5 : 0];
        const CUtensorMap* bmap0 = &maps.m[ti.extra ? 6 : 1];
        // weights are kept in L2 when other token tiles read them again (the
        // expert's next token tile; every token tile of the extra problem)
        const bool wshared =
            ti.extra ? p.rows_x > S::kTokens
                     : ti.act0 + S::kTokens < epoff[ti.expert] + ecount[ti.expert];
        const uint64_t pa = wshared ? pol_keep : pol_stream;
        for (int kb = 0; kb < ti.kblocks; kb += S::kAtoms) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, 0x2100 + stage)) { ok = false; break; }
          uint8_t* sa = smem + stage * S::kStageBytes;
          uint8_t* sb = sa + S::kAtoms * S::kABytes;
          const int na = min(S::kAtoms, ti.kblocks - kb);   // K atoms in this stage
          if (leader) mbar_arrive_expect_tx(&full[stage], na * (2 * S::kABytes + ti.n * 128));
          const uint32_t bar = cluster_map(smem_u32(&full[stage]), 0);
          const int kg = ti.extra ? p.kgroup_x : 0;   // K split over the weight tensor's groups
          for (int q = 0; q < na; ++q) {
            const int k = (kb + q) * 64;
            tma_load_3d_pair(sa + q * S::kABytes, amap, bar, kg ? k % kg : k, ti.w0 + static_cast<int>(rank) * 128,
                             kg ? k / kg : ti.expert, pa);
            int done = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int box = 128 >> i;
              if (half - done >= box) {
                tma_load_3d_pair(sb + q * S::kBBytes + done * 128, bmap0 + i, bar, k, b_row0 + done, 0, pol_norm);
                done += box;
              }
            }
          }
          issued = true;
          if (++stage == S::kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (*abort_flag && issued) {
        // loads in flight complete on the even CTA's barrier; give them time to
        // land before this CTA's shared memory can go away
        const long long t0 = clock64();
        while (clock64() - t0 < (1LL << 22)) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (even CTA) ----------------
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true, any = false;
      for (int t = cluster; t < ntiles && ok; t += nclusters) {
        const Tile2 ti = tc2_tile(p, t, ntiles, nextra, prefix, ecount, epoff);
        if (!ti.valid) continue;
        const int acc = local & 1;
        if (!mbar_wait(&tempty[acc], ((local >> 1) & 1) ^ 1, abort_flag, p.err, 0x2200 + acc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256;
        const uint32_t idesc = idesc_bf16_f32(256, ti.n);
        for (int kb = 0; kb < ti.kblocks; kb += S::kAtoms) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, 0x2300 + stage)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * S::kStageBytes);
          const uint32_t sb = sa + S::kAtoms * S::kABytes;
          const int na = min(S::kAtoms, ti.kblocks - kb);
          for (int q = 0; q < na; ++q)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_pair(d_tmem, sdesc_kmajor_sw128(sa + q * S::kABytes + kk * 32),
                            sdesc_kmajor_sw128(sb + q * S::kBBytes + kk * 32), idesc, (kb | q | kk) != 0 ? 1u : 0u);
          any = true;
          mma_commit_pair(&empty[stage], 0x3);
          if (++stage == S::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit_pair(&tfull[acc], 0x3);
        ++local;
      }
      if (any) {
        mma_commit_pair(drain, 0x1);
        const long long t0 = clock64();
        while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitLimitCycles / 4) {}
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5, both CTAs) ----------------
    const int q = warp & 3;        // TMEM lane quarter: feature rows q * 32 .. q * 32 + 31 of the CTA's 128
    int local = 0;
    for (int t = cluster; t < ntiles; t += nclusters) {
      const Tile2 ti = tc2_tile(p, t, ntiles, nextra, prefix, ecount, epoff);
      if (!ti.valid) continue;
      const int acc = local & 1;
      const float* const row_scale = ti.extra ? nullptr : p.row_scale;
      // the gates of the tile's tokens, all requested at once and before the
      // wait for the accumulator (lane: token c * 32 + lane of chunk c), so
      // their latency hides behind the tile's MMAs
      float gates[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int tk = c * 32 + lane;
        gates[c] = (EPI == EPI_GATE && row_scale && tk < ti.act_n) ? __ldg(row_scale + ti.act0 + tk) : 1.0f;
      }
      if (!mbar_wait(&tfull[acc], (local >> 1) & 1, abort_flag, p.err, 0x2400 + acc)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * 256;
      const int wbase = ti.w0 + static_cast<int>(rank) * 128;
      const uint64_t pol_out = policy_evict_first();   // outputs stream out; the next kernel reads them from HBM
      const int cols = ti.extra ? p.cols_x : p.cols;
      __nv_bfloat16* const out = reinterpret_cast<__nv_bfloat16*>(ti.extra ? p.out_x : p.out);
      const long long ld_out = ti.extra ? p.ld_out_x : p.ld_out;
      const int nchunks = (ti.act_n + 31) / 32;
      __nv_bfloat16* tb = epi_tile + q * 32 * 32;
      // this lane owns feature wbase + r for 32 tokens a chunk; each warp's
      // 32 x 32 block is transposed through shared memory so each token's 32
      // features go out as 16-byte stores
      auto emit = [&](int c, const uint32_t (&v)[32], float gate) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float val = __uint_as_float(v[j]);
          if (EPI == EPI_SQRELU) {
            val = fmaxf(val, 0.0f);
            val = val * val;
          } else if (EPI == EPI_GATE) {
            val = val * __shfl_sync(0xffffffffu, gate, j);
          }
          tb[j * 32 + lane] = __float2bfloat16_rn(val);
        }
        __syncwarp();
        const int seg = lane & 3;
        const int col0 = wbase + q * 32 + seg * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = (lane >> 2) + 8 * i;
          const int tok = c * 32 + j;
          if (tok < ti.act_n && col0 < cols) {
            const uint4 u = *reinterpret_cast<const uint4*>(tb + j * 32 + seg * 8);
            st_global_v4_hint(out + (ti.act0 + tok) * ld_out + col0, u, pol_out);
          }
        }
        __syncwarp();
      };
      // two chunks per tensor-memory wait
#pragma unroll
      for (int c = 0; c < 8; c += 2) {
        if (c >= nchunks) break;
        uint32_t v0[32], v1[32];
        tmem_ld_32x32b_x32(t_row + c * 32, v0);
        if (c + 1 < nchunks) tmem_ld_32x32b_x32(t_row + (c + 1) * 32, v1);
        tmem_ld_wait();
        emit(c, v0, gates[c]);
        if (c + 1 < nchunks) emit(c + 1, v1, gates[c + 1]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_map(smem_u32(&tempty[acc]), 0));
      ++local;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_barrier();   // the pair's MMAs, loads and epilogues are all done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, S::kTmemCols);
  }
}

}  // namespace lmoe
