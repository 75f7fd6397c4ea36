// Grouped block-scaled NVFP4 expert GEMM on CTA pairs, weight-major
// (tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16, M = 256):
//
//   D[w, t] = sum_k (q_w[w,k] s_w[w,k/16]) (q_a[t,k] s_a[t,k/16])
//     w: 256 output features of expert e (128 per CTA of the pair)
//     t: up to 128 of the expert's tokens (the MMA's N, 64 or 128)
//
// Each CTA loads its 128 weight rows and their scales, its half of the token
// rows, and the scales of all N tokens (the pair's MMA reads B's scales in
// both CTAs); every load is a TMA load with .cta_group::2 that completes on
// the even CTA's barrier (no multicast). The even CTA's single MMA thread
// moves the scales to both CTAs' tensor memory with tcgen05.cp.cta_group::2
// and issues the pair's MMAs.
//
// Tensor memory per CTA: two accumulators of 128 columns ([0,128) and
// [128,256)), so the MMAs of a tile wait only for the epilogue of the tile
// two before it; scales at [256, 288): 4 x 4 columns of weight scales and
// 4 x 4 of token scales per stage. (An FP4 tile of 256 tokens would need two
// 256-column accumulators and leave no columns for the scales; letting them
// overlap made every tile's MMAs wait for the previous tile's epilogue, and
// with FP4's short tiles that wait was most of the time.)
// Epilogue: eight warps, two per TMEM lane quarter (one feature per lane),
// each reading its two 32-token chunks with one wait and releasing the
// accumulator before any arithmetic; a chunk is transposed through shared
// memory so that each lane then holds one token's 32 features:
//   GEMM 1: a = relu(acc * s_z * s_w1[e])^2 quantised to NVFP4 with the static
//           scale s_a (16-feature blocks along the token's row)
//   GEMM 2: y = acc * s_a * s_w2[e] * gate[token], BF16
// No TMA load here uses cluster multicast.
#pragma once

#include "gemm_fp4.cuh"
#include "gemm_tc2.cuh"

namespace lmoe {

struct Fp4pSmem {
  static constexpr int kA = 128 * 128;        // 128 weight rows x 256 fp4
  static constexpr int kB = 64 * 128;         // up to 64 token rows (this CTA's half) x 256 fp4
  static constexpr int kSFA = 4 * 512;        // 4 atoms (4 K-groups of 64) of this CTA's 128 weight rows
  static constexpr int kSFB = 4 * 512;        // 4 atoms of the tile's (up to) 128 tokens
  static constexpr int kStage = kA + kB + kSFA + kSFB;   // 28672 = 28 KB, a multiple of 1024
  static constexpr int kStages = 6;
  static constexpr int kBarOffset = kStages * kStage;
  static constexpr int kMaxGroups = 1024;
  static constexpr int kPrefixOffset = kBarOffset + 256;
  static constexpr int kEpiOffset = (kPrefixOffset + (kMaxGroups + 1) * 4 + 15) / 16 * 16;
  static constexpr int kEpiPitch = 33;        // floats per transposed row (bank-conflict free)
  static constexpr int kEpiWarpBytes = 32 * kEpiPitch * 4;
  // per expert: row count and first padded row (read from global memory once)
  static constexpr int kExpertOffset = kEpiOffset + 8 * kEpiWarpBytes;
  static constexpr int kBytes = kExpertOffset + 2 * kMaxGroups * 4 + 1024;
  static constexpr int kThreads = 64 + 256;   // producer, MMA, eight epilogue warps
  static constexpr int kAccCols = 128;        // accumulator b at columns [128 b, 128 b + 128)
  static constexpr int kSfaCol = 256;
  static constexpr int kSfbCol = 272;
  static constexpr int kTokens = 128;
};

struct Fp4pParams {
  int rows;                   // padded token rows (a multiple of 128)
  int cols;                   // output features per expert (a multiple of 256)
  int kblocks;                // 256-element K blocks
  int groups64;               // K / 64
  const int* offsets;
  const int* padded_offsets;
  int groups;
  const float* in_scale;      // global scale of the tokens (device scalar, or [groups] with in_scale_grouped)
  int in_scale_grouped;
  const float* w_scale;       // [groups] global scales of the weights
  const float* out_scale;     // GEMM1: static global scale of a (device scalar)
  const float* row_scale;     // GEMM2: gate per padded row (nullable)
  void* out;                  // GEMM1: codes [rows][cols/2]; GEMM2: bf16 [rows][ld_out]
  uint8_t* out_sf;            // GEMM1: MMA-tiled scales of a
  long long ld_out;
  DevErr err;
};

// Tensor maps: [0] weight codes [groups][cols][K/2] (128-row boxes),
// [1..4] token codes [rows][K/2] with boxes of 128, 64, 32, 16 rows,
// [5] weight scales [groups][cols/128 * K/64 * 2][256 B] (8-row boxes = 4 atoms),
// [6] token scales [rows/128 * K/64 * 2][256 B] (8-row boxes).
struct Fp4pMaps {
  CUtensorMap m[7];
};

// Scale atom -> tensor memory of both CTAs of the pair (each from its own
// shared memory at the same offset).
__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mma_nvfp4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

struct Tile4p {
  int valid;
  int expert;
  int act0;    // first padded token row of the tile
  int act_n;   // tokens in the tile
  int w0;      // first feature of the pair's 256
  int n;       // MMA N: act_n rounded up to 64
};

// Pair tile t: expert e, token tile tt (128 tokens), weight tile of 256
// features; the weight tiles of one token tile are consecutive.
__device__ __forceinline__ Tile4p fp4p_tile(const Fp4pParams& p, int t, const int* prefix, const int* ecount,
                                            const int* epoff) {
  Tile4p ti;
  const int ntw = p.cols / 256;
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
  ti.act0 = epoff[e] + tt * Fp4pSmem::kTokens;
  ti.act_n = min(Fp4pSmem::kTokens, n_e - tt * Fp4pSmem::kTokens);
  ti.valid = ti.act_n > 0;
  // the MMA's N: 64 or 128 (the token scales sit in one 128-row atom)
  ti.n = ti.act_n <= 64 ? 64 : 128;
  return ti;
}

template <int EPI>
__global__ void __launch_bounds__(Fp4pSmem::kThreads, 1)
    fp4p_gemm_kernel(const __grid_constant__ Fp4pMaps maps, const Fp4pParams p) {
  pdl_begin();
  using S = Fp4pSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOffset);
  uint64_t* empty = full + S::kStages;
  uint64_t* tfull = empty + S::kStages;   // [2]
  uint64_t* tempty = tfull + 2;           // [2], even CTA: both CTAs' 16 epilogue warps arrive
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_ptr + 1);
  int* prefix = reinterpret_cast<int*>(smem + S::kPrefixOffset);
  float* epi = reinterpret_cast<float*>(smem + S::kEpiOffset);
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
    const int ntw = p.cols / 256;
    for (int e = threadIdx.x; e < p.groups; e += blockDim.x) {
      int n_e = __ldg(p.offsets + e + 1) - __ldg(p.offsets + e);
      if (kChecks) {   // the expert's rows must fit its padded range inside the buffer
        const int ps = __ldg(p.padded_offsets + e), pe = __ldg(p.padded_offsets + e + 1);
        if (n_e < 0 || ps < 0 || pe > p.rows || ps + n_e > pe) {
          dev_report(p.err, kErrBounds, 0x5400);
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
      mbar_init(&tempty[a], 16);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    for (int i = 0; i < 7; ++i) tma_prefetch_desc(&maps.m[i]);
  }
  if (warp == 1) tmem_alloc_pair(tmem_ptr, 512);
  tc_fence_before();
  __syncthreads();
  cluster_barrier();   // both CTAs' barriers and TMEM exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_ptr;
  const int ntiles = prefix[p.groups];

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      const uint64_t pol = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int t = cluster; t < ntiles && ok; t += nclusters) {
        const Tile4p ti = fp4p_tile(p, t, prefix, ecount, epoff);
        if (!ti.valid) continue;
        const int half = ti.n >> 1;
        const int b_row0 = ti.act0 + static_cast<int>(rank) * half;
        const int rb_w = (ti.w0 >> 7) + static_cast<int>(rank);   // this CTA's weight row block
        const int rb_t = ti.act0 >> 7;                              // the tile's token row block
        const uint32_t stage_bytes = 2u * (S::kA + S::kSFA + S::kSFB) + static_cast<uint32_t>(ti.n) * 128u;
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, 0x1500 + stage)) { ok = false; break; }
          uint8_t* sa = smem + stage * S::kStage;
          uint8_t* sb = sa + S::kA;
          uint8_t* ssfa = sb + S::kB;
          uint8_t* ssfb = ssfa + S::kSFA;
          if (leader) mbar_arrive_expect_tx(&full[stage], stage_bytes);
          const uint32_t bar = cluster_map(smem_u32(&full[stage]), 0);
          tma_load_3d_pair(sa, &maps.m[0], bar, kb * 128, ti.w0 + static_cast<int>(rank) * 128, ti.expert, pol);
          // half is 32 or 64 rows: maps 2 (64-row boxes) and 3 (32-row boxes)
          tma_load_3d_pair(sb, &maps.m[half == 64 ? 2 : 3], bar, kb * 128, b_row0, 0, pol);
          // scale atoms (4 per row block and K block) as 8 rows of 256 bytes; every
          // map here is three-dimensional, the token maps with one group
          tma_load_3d_pair(ssfa, &maps.m[5], bar, 0, (rb_w * p.groups64 + kb * 4) * 2, ti.expert, pol);
          tma_load_3d_pair(ssfb, &maps.m[6], bar, 0, (rb_t * p.groups64 + kb * 4) * 2, 0, pol);
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
      const uint32_t sfa_t = tmem_base + S::kSfaCol;
      const uint32_t sfb_t = tmem_base + S::kSfbCol;
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true, any = false;
      for (int t = cluster; t < ntiles && ok; t += nclusters) {
        const Tile4p ti = fp4p_tile(p, t, prefix, ecount, epoff);
        if (!ti.valid) continue;
        const int acc = local & 1;
        if (!mbar_wait(&tempty[acc], ((local >> 1) & 1) ^ 1, abort_flag, p.err, 0x1600 + acc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * S::kAccCols;
        const uint32_t idesc = idesc_nvfp4(256, ti.n);
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, 0x1700 + stage)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_s = smem_u32(smem + stage * S::kStage);
          const uint32_t b_s = a_s + S::kA;
          const uint32_t sfa_s = b_s + S::kB;
          const uint32_t sfb_s = sfa_s + S::kSFA;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            tmem_cp_sf_pair(sfa_t + kk * 4, sdesc_sf_atom(sfa_s + kk * 512));
            tmem_cp_sf_pair(sfb_t + kk * 4, sdesc_sf_atom(sfb_s + kk * 512));
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_nvfp4_pair(d_tmem, sdesc_kmajor_sw128(a_s + kk * 32), sdesc_kmajor_sw128(b_s + kk * 32), idesc,
                           sfa_t + kk * 4, sfb_t + kk * 4, (kb | kk) != 0 ? 1u : 0u);
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
  } else if (warp >= 2) {
    // ---------------- epilogue (warps 2..9, both CTAs) ----------------
    const int q = warp & 3;             // TMEM lane quarter
    const int half = (warp - 2) >> 2;   // which two of the four 32-token chunks
    float* tb = epi + (warp - 2) * (S::kEpiWarpBytes / 4);
    const float in_s0 = __ldg(p.in_scale);
    const float out_s = (EPI == FP4_EPI_SQRELU_QUANT) ? __ldg(p.out_scale) : 0.0f;
    const int groups64_out = p.cols / 64;
    const uint64_t pol_out = policy_evict_first();
    int local = 0;
    for (int t = cluster; t < ntiles; t += nclusters) {
      const Tile4p ti = fp4p_tile(p, t, prefix, ecount, epoff);
      if (!ti.valid) continue;
      const int buf = local & 1;
      const float in_s = p.in_scale_grouped ? __ldg(p.in_scale + ti.expert) : in_s0;
      const float scale = __fmul_rn(in_s, __ldg(p.w_scale + ti.expert));
      const int f0 = ti.w0 + static_cast<int>(rank) * 128 + q * 32;   // first feature of this warp
      // GEMM 2: the gates of this warp's two chunks (chunk half * 2 + i, token
      // (half * 2 + i) * 32 + lane), requested before the accumulator wait
      float gates[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int tk = (half * 2 + i) * 32 + lane;
        gates[i] = (EPI == FP4_EPI_GATE_BF16 && p.row_scale && tk < ti.act_n) ? __ldg(p.row_scale + ti.act0 + tk)
                                                                                : 1.0f;
      }
      if (!mbar_wait(&tfull[buf], (local >> 1) & 1, abort_flag, p.err, 0x1800 + buf)) break;
      tc_fence_after();
      const uint32_t acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * S::kAccCols;
      // chunk c (32 tokens): transpose so that lane j holds token c*32+j's 32 features
      auto emit = [&](int c, const uint32_t (&v)[32], float g) {
        if (c * 32 >= ti.act_n) return;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float h = __uint_as_float(v[j]) * scale;
          if (EPI == FP4_EPI_SQRELU_QUANT) {
            h = fmaxf(h, 0.0f);
            h = h * h;
          }
          tb[j * S::kEpiPitch + lane] = h;
        }
        __syncwarp();
        float x[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = tb[lane * S::kEpiPitch + i];
        __syncwarp();
        const int tok = c * 32 + lane;
        if (tok >= ti.act_n) return;
        const long long row = ti.act0 + tok;
        if (EPI == FP4_EPI_SQRELU_QUANT) {
          uint2 c0, c1;
          const uint32_t s0 = fp4_quant16(x, out_s, c0);
          const uint32_t s1 = fp4_quant16(x + 16, out_s, c1);
          uint8_t* codes = reinterpret_cast<uint8_t*>(p.out) + row * (p.cols / 2) + f0 / 2;
          st_global_v4_hint(codes, make_uint4(c0.x, c0.y, c1.x, c1.y), pol_out);
          const int j0 = f0 / 16;
          p.out_sf[fp4_sf_offset(row, j0, groups64_out)] = static_cast<uint8_t>(s0);
          p.out_sf[fp4_sf_offset(row, j0 + 1, groups64_out)] = static_cast<uint8_t>(s1);
        } else {
          __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + row * p.ld_out + f0;
#pragma unroll
          for (int j = 0; j < 32; j += 16) {
            uint32_t u[8];
#pragma unroll
            for (int h = 0; h < 8; ++h) u[h] = pack_bf16x2(x[j + 2 * h] * g, x[j + 2 * h + 1] * g);
            st_global_v8_hint(o + j, u, pol_out);
          }
        }
      };
      // both chunks with one wait, then the accumulator goes back to the MMA
      // (on the even CTA's barrier) before any arithmetic
      const int nch = (ti.act_n + 31) / 32;
      const int c = half * 2;
      uint32_t v0[32], v1[32];
      if (c < nch) tmem_ld_32x32b_x32(acc + c * 32, v0);
      if (c + 1 < nch) tmem_ld_32x32b_x32(acc + (c + 1) * 32, v1);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_map(smem_u32(&tempty[buf]), 0));
      emit(c, v0, gates[0]);
      emit(c + 1, v1, gates[1]);
      ++local;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_barrier();   // the pair's MMAs, loads and epilogues are all done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace lmoe
