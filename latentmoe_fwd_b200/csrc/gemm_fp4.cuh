// Grouped block-scaled NVFP4 GEMM for sm_100a (tcgen05.mma kind::mxf4nvf4,
// 16-element blocks with E4M3 scales), used for the routed experts when the
// expert weights and the latent activations are NVFP4:
//
//   acc[r, c] = sum_k (q_a[r,k] * sa[r,k/16]) * (q_w[c,k] * sw[c,k/16])
//   GEMM 1: a = relu(acc * s_z * s_w1[e])^2, quantised to NVFP4 with the
//           static scale s_a (codes + MMA-tiled scales written directly)
//   GEMM 2: y = acc * s_a * s_w2[e] * gate[row], stored as BF16
//
// Structure as the BF16 kernel (TMA producer warp, single-thread MMA issuer,
// persistent tiles of 128 activation rows x 256 output features), but with
// eight epilogue warps -- two per TMEM lane quarter, each draining half of the
// columns -- because quantising a in GEMM 1 costs more than the MMAs; plus:
//  * each stage carries the tile's scale atoms (512 B = 128 rows x 4 scales),
//    fetched with bulk copies and moved shared -> tensor memory with
//    tcgen05.cp (32 lanes x 128 bit, replicated over the four lane quarters)
//    just before the MMAs that read them; copies and MMAs issued by one
//    thread execute in order, so one scale buffer in TMEM suffices;
//  * the two 256-column accumulators overlap in TMEM columns [192, 256) to
//    leave room for the scales ([0,256) and [192,448); scales at 448+); the
//    epilogue drains that shared slice first and then releases the MMA.
#pragma once

#include "lmoe_device.cuh"

namespace lmoe {

// FP4_EPI_F32: out = acc * scales in fp32 (the training recipe's backward
// feeds such results to its stochastic quantisers, which need them unrounded)
enum Fp4Epi : int { FP4_EPI_SQRELU_QUANT = 0, FP4_EPI_GATE_BF16 = 1, FP4_EPI_F32 = 2 };

struct Fp4Params {
  int rows;                   // padded rows of A (a multiple of 128)
  int cols;                   // output features per expert
  int kblocks;                // 256-element K blocks
  int sf_groups_a;            // K / 64: scale atoms per 128-row block of A
  int sf_groups_b;            // K / 64 for B
  const uint8_t* sfa;         // activation scales, MMA-tiled over the padded rows
  const uint8_t* sfb;         // weight scales, MMA-tiled, expert-major
  long long sfb_expert_bytes; // bytes of one expert's weight scales
  const int* offsets;
  const int* padded_offsets;
  int groups;
  const float* in_scale;      // global scale of A (device scalar, or [groups] with in_scale_grouped)
  int in_scale_grouped;
  const float* w_scale;       // [groups] global scales of B
  const float* out_scale;     // GEMM1: static global scale of a (device scalar)
  const float* row_scale;     // GEMM2: gate per padded row (nullable)
  void* out;                  // GEMM1: codes [rows][cols/2]; GEMM2: bf16 [rows][cols]
  uint8_t* out_sf;            // GEMM1: MMA-tiled scales of a
  long long ld_out;           // GEMM2: elements per row
  int out_vec32;              // GEMM2: rows start on 32-byte boundaries (32-byte stores)
  // K-batched problems (the kernel's BATCH form): group g multiplies K
  // columns [kgroup_tab[2g], + 256 * kgroup_tab[2g+1]) of A [rows][K] and of
  // B [cols][K] (shared matrices, K the sum over groups) into its own output
  // at out + g * out_group_stride
  const int* kgroup_tab;
  long long out_group_stride;
  DevErr err;
};

struct Fp4Smem {
  static constexpr int kA = 128 * 128;       // 128 rows x 256 fp4
  static constexpr int kB = 256 * 128;       // 256 rows x 256 fp4
  static constexpr int kSFA = 4 * 512;       // 4 atoms (4 K-blocks of 64) x 128 rows
  static constexpr int kSFB = 8 * 512;       // 4 K-blocks x 2 row blocks
  static constexpr int kStage = kA + kB + kSFA + kSFB;   // 55296
  static constexpr int kStages = 4;
  static constexpr int kBarOffset = kStages * kStage;
  static constexpr int kMaxGroups = 1024;
  // per-expert padded start and real end rows, copied once per CTA so that
  // the tile -> expert lookup is a short walk in shared memory
  static constexpr int kRowsOffset = kBarOffset + 256;
  static constexpr int kBytes = kRowsOffset + 2 * (kMaxGroups + 1) * 4 + 1024;
  static constexpr int kThreads = 64 + 256;   // producer, MMA, eight epilogue warps
  static constexpr int kAccCols = 256;
  static constexpr int kAcc1 = 192;          // second accumulator starts here
  static constexpr int kSfaCol = 448;
  static constexpr int kSfbCol = 464;
};

__host__ __device__ constexpr uint32_t idesc_nvfp4(int M, int N) {
  return (1u << 7)                                   // A format E2M1
         | (1u << 10)                                // B format E2M1
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (0u << 23)                                // scale format UE4M3
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory descriptor of one 512-byte scale atom (32 rows x 16 B, no
// swizzle; 8-row core matrices 128 B apart) as the source of tcgen05.cp.
__device__ __forceinline__ uint64_t sdesc_sf_atom(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(128 >> 4) << 16;     // leading byte offset
  d |= static_cast<uint64_t>(128 >> 4) << 32;     // stride byte offset (next 8 rows)
  d |= static_cast<uint64_t>(1) << 46;            // version
  return d;                                       // swizzle none
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mma_nvfp4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// E4M3 scale of a block and its exact value (see the quantiser).
__device__ __forceinline__ uint32_t fp4_cvt_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

__device__ __forceinline__ float fp4_e4m3_value(uint32_t c) {
  const int e = (c >> 3) & 15, f = c & 7;
  return e == 0 ? ldexpf(static_cast<float>(f), -9) : ldexpf(static_cast<float>(8 + f), e - 10);
}

// Quantise 16 values with global scale s_g: returns the E4M3 code and 8 code bytes.
__device__ __forceinline__ uint32_t fp4_quant16(const float* x, float s_g, uint2& codes) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const uint32_t sb = fp4_cvt_e4m3(__fdiv_rn(amax, __fmul_rn(s_g, 6.0f)));
  const float dec = fp4_e4m3_value(sb);
  codes.x = 0;
  codes.y = 0;
  if (dec != 0.0f) {
    const float sc = __fmul_rn(dec, s_g);
    codes = e2m1_codes16(x, sc, __frcp_rn(sc));
  }
  return sb;
}

__device__ __forceinline__ long long fp4_sf_offset(long long row, int j, int groups64) {
  return ((row >> 7) * groups64 + (j >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (j & 3);
}

template <int EPI, bool BATCH = false>
__global__ void __launch_bounds__(Fp4Smem::kThreads, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmA32, const Fp4Params p) {
  pdl_begin();
  using S = Fp4Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOffset);
  uint64_t* empty = full + S::kStages;
  uint64_t* tfull = empty + S::kStages;   // [2]
  uint64_t* overlap_free = tfull + 2;     // [1]: previous tile drained the shared slice
  uint64_t* drain = overlap_free + 1;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_ptr + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&tfull[0], 1);
    mbar_init(&tfull[1], 1);
    mbar_init(overlap_free, 8);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmA32);
    tma_prefetch_desc(&tmB);
  }
  int* s_pstart = reinterpret_cast<int*>(smem + S::kRowsOffset);   // [groups + 1] padded starts
  int* s_rend = s_pstart + S::kMaxGroups + 1;                          // [groups] real ends
  // BATCH: s_pstart[g] = first K column of group g, s_rend[g] = its K blocks
  for (int g = threadIdx.x; BATCH && g < p.groups; g += blockDim.x) {
    int k0 = __ldg(p.kgroup_tab + 2 * g), nk = __ldg(p.kgroup_tab + 2 * g + 1);
    if (kChecks && (k0 < 0 || (k0 & 255) || nk < 0 || k0 / 256 + nk > p.kblocks)) {   // within K
      dev_report(p.err, kErrBounds, 0x5302);
      k0 = 0;
      nk = 0;
    }
    s_pstart[g] = k0;
    s_rend[g] = nk;
  }
  for (int g = threadIdx.x; !BATCH && g <= p.groups; g += blockDim.x) {
    int ps = __ldg(p.padded_offsets + g);
    if (kChecks && (ps < 0 || ps > p.rows || (ps & 127))) {
      dev_report(p.err, kErrBounds, 0x5300);
      ps = p.rows;
    }
    s_pstart[g] = ps;
    if (g < p.groups) {
      int n_e = __ldg(p.offsets + g + 1) - __ldg(p.offsets + g);
      if (kChecks) {   // the expert's rows must fit its padded range
        const int pe = __ldg(p.padded_offsets + g + 1);
        if (n_e < 0 || pe < ps || pe > p.rows || ps + n_e > pe) {
          dev_report(p.err, kErrBounds, 0x5301);
          n_e = 0;
        }
      }
      s_rend[g] = ps + n_e;
    }
  }
  if (warp == 1) tmem_alloc(tmem_ptr, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_ptr;

  const int ntw = (p.cols + 255) / 256;
  const int tpg = (p.rows >> 7) * ntw;   // BATCH: tiles per group
  const int ntiles = BATCH ? p.groups * tpg : (s_pstart[p.groups] >> 7) * ntw;

  // a CTA visits its tiles in increasing order, so the owning expert (the
  // largest e with padded start <= act0) only moves forward. nkb: the tile's
  // 256-element K blocks from K column koff.
  int cur_e = 0;
  auto tile_of = [&](int t, int& e, int& act0, int& act_n, int& w0, int& nkb, int& koff) {
    if (BATCH) {
      e = t / tpg;
      const int rem = t - e * tpg;
      w0 = (rem % ntw) * 256;
      act0 = (rem / ntw) * 128;
      koff = s_pstart[e];
      nkb = s_rend[e];
      act_n = nkb > 0 ? 128 : 0;
    } else {
      w0 = (t % ntw) * 256;
      act0 = (t / ntw) * 128;
      while (cur_e + 1 < p.groups && s_pstart[cur_e + 1] <= act0) ++cur_e;
      e = cur_e;
      act_n = min(128, s_rend[e] - act0);
      nkb = p.kblocks;
      koff = 0;
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_normal();   // read again by the expert's other row tiles
      const uint64_t pol_a = policy_evict_last();     // read by every column tile
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, last_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int e, act0, act_n, w0, nkb, koff;
        tile_of(t, e, act0, act_n, w0, nkb, koff);
        if (act_n <= 0) continue;
        const uint8_t* sfa_blk = p.sfa + (static_cast<long long>(act0 >> 7) * p.sf_groups_a + koff / 64) * 512;
        const uint8_t* sfb_e = p.sfb + static_cast<long long>(e) * p.sfb_expert_bytes + (koff / 64) * 512;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, 0x1100 + stage)) { ok = false; break; }
          uint8_t* sa = smem + stage * S::kStage;
          uint8_t* sb = sa + S::kA;
          uint8_t* ssfa = sb + S::kB;
          uint8_t* ssfb = ssfa + S::kSFA;
          // a tile of at most 32 real rows (decode) loads only those 32 rows of
          // A: the MMA's other rows read stale codes, but an output row reads
          // only its own A row and the epilogue stores real rows only
          const bool thin = act_n <= 32;
          mbar_arrive_expect_tx(&full[stage], thin ? S::kStage - S::kA + 32 * 128 : S::kStage);
          tma_load_3d(sa, thin ? &tmA32 : &tmA, &full[stage], koff / 2 + kb * 128, act0, 0, pol_a);
          tma_load_3d(sb, &tmB, &full[stage], koff / 2 + kb * 128, w0, BATCH ? 0 : e, pol_w);
          bulk_load(ssfa, sfa_blk + kb * 4 * 512, S::kSFA, &full[stage]);
#pragma unroll
          for (int nb = 0; nb < 2; ++nb)
            bulk_load(ssfb + nb * 2048,
                      sfb_e + (static_cast<long long>((w0 >> 7) + nb) * p.sf_groups_b + kb * 4) * 512, 2048,
                      &full[stage]);
          issued_mask |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S::kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < S::kStages; ++s)
          if (issued_mask & (1u << s)) {
            long long t0 = clock64();
            while (!mbar_try_wait(&full[s], (last_par >> s) & 1) && clock64() - t0 < kWaitLimitCycles / 4) {}
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_nvfp4(128, 256);
      const uint32_t sfa_t = tmem_base + S::kSfaCol;
      const uint32_t sfb_t = tmem_base + S::kSfbCol;
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true, any = false;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int e, act0, act_n, w0, nkb, koff;
        tile_of(t, e, act0, act_n, w0, nkb, koff);
        if (act_n <= 0) continue;
        if (local > 0) {
          if (!mbar_wait(overlap_free, (local - 1) & 1, abort_flag, p.err, 0x1200)) { ok = false; break; }
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ((local & 1) ? S::kAcc1 : 0);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, 0x1300 + stage)) { ok = false; break; }
          tc_fence_after();
          uint8_t* sa = smem + stage * S::kStage;
          const uint32_t a_s = smem_u32(sa);
          const uint32_t b_s = a_s + S::kA;
          const uint32_t sfa_s = b_s + S::kB;
          const uint32_t sfb_s = sfa_s + S::kSFA;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            tmem_cp_sf(sfa_t + kk * 4, sdesc_sf_atom(sfa_s + kk * 512));
            tmem_cp_sf(sfb_t + kk * 8, sdesc_sf_atom(sfb_s + kk * 512));
            tmem_cp_sf(sfb_t + kk * 8 + 4, sdesc_sf_atom(sfb_s + 2048 + kk * 512));
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_nvfp4(d_tmem, sdesc_kmajor_sw128(a_s + kk * 32), sdesc_kmajor_sw128(b_s + kk * 32), idesc,
                      sfa_t + kk * 4, sfb_t + kk * 8, (kb | kk) != 0 ? 1u : 0u);
          }
          any = true;
          mma_commit(&empty[stage]);
          if (++stage == S::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(&tfull[local & 1]);
        ++local;
      }
      if (any) {
        mma_commit(drain);
        long long t0 = clock64();
        while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitLimitCycles / 4) {}
      }
    }
  } else {
    const int q = warp & 3;             // TMEM lane quarter
    const int half = (warp - 2) >> 2;   // which four of the eight 32-column chunks
    const int r = q * 32 + lane;
    int local = 0;
    const float in_s0 = __ldg(p.in_scale);
    const float out_s = (EPI == FP4_EPI_SQRELU_QUANT) ? __ldg(p.out_scale) : 0.0f;
    const int groups64_out = (p.cols + 63) / 64;
    const uint64_t pol_out = policy_evict_first();
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      int e, act0, act_n, w0, nkb, koff;
      tile_of(t, e, act0, act_n, w0, nkb, koff);
      if (act_n <= 0) continue;
      const long long obase = BATCH ? e * p.out_group_stride : 0;
      const int buf = local & 1;
      const long long row = act0 + r;
      const bool row_ok = r < act_n;
      // per-tile scalars fetched before the accumulator is ready
      const float gate = (EPI != FP4_EPI_SQRELU_QUANT && p.row_scale && row_ok) ? __ldg(p.row_scale + row) : 1.0f;
      const float in_s = p.in_scale_grouped ? __ldg(p.in_scale + e) : in_s0;
      const float scale = __fmul_rn(in_s, __ldg(p.w_scale + e));
      if (!mbar_wait(&tfull[buf], (local >> 1) & 1, abort_flag, p.err, 0x1400 + buf)) break;
      tc_fence_after();
      const uint32_t acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + (buf ? S::kAcc1 : 0);
      auto release = [&]() {   // this warp no longer reads the TMEM slice the next tile overwrites
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(overlap_free);
      };
      auto emit = [&](int c, const uint32_t (&v)[32]) {
        const int col0 = w0 + c * 32;
        if (!row_ok || col0 >= p.cols) return;
        if (EPI == FP4_EPI_SQRELU_QUANT) {
          float a[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float h = fmaxf(__uint_as_float(v[j]) * scale, 0.0f);
            a[j] = h * h;
          }
          uint2 c0, c1;
          const uint32_t s0 = fp4_quant16(a, out_s, c0);
          const uint32_t s1 = fp4_quant16(a + 16, out_s, c1);
          uint8_t* codes = reinterpret_cast<uint8_t*>(p.out) + row * (p.cols / 2) + col0 / 2;
          st_global_v4_hint(codes, make_uint4(c0.x, c0.y, c1.x, c1.y), pol_out);
          const int j0 = col0 / 16;
          p.out_sf[fp4_sf_offset(row, j0, groups64_out)] = static_cast<uint8_t>(s0);
          p.out_sf[fp4_sf_offset(row, j0 + 1, groups64_out)] = static_cast<uint8_t>(s1);
        } else if (EPI == FP4_EPI_F32) {
          float* o = reinterpret_cast<float*>(p.out) + obase + row * p.ld_out + col0;
          const float sg = scale * gate;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(o + j) =
                make_float4(__uint_as_float(v[j]) * sg, __uint_as_float(v[j + 1]) * sg,
                            __uint_as_float(v[j + 2]) * sg, __uint_as_float(v[j + 3]) * sg);
        } else {
          __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + obase + row * p.ld_out + col0;
          const float sg = scale * gate;
          if (p.out_vec32) {   // whole 32-byte sectors per store
#pragma unroll
            for (int j = 0; j < 32; j += 16) {
              uint32_t u[8];
#pragma unroll
              for (int h = 0; h < 8; ++h)
                u[h] = pack_bf16x2(__uint_as_float(v[j + 2 * h]) * sg, __uint_as_float(v[j + 2 * h + 1]) * sg);
              st_global_v8_hint(o + j, u, pol_out);
            }
            return;
          }
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(v[j + 0]) * sg, __uint_as_float(v[j + 1]) * sg);
            u.y = pack_bf16x2(__uint_as_float(v[j + 2]) * sg, __uint_as_float(v[j + 3]) * sg);
            u.z = pack_bf16x2(__uint_as_float(v[j + 4]) * sg, __uint_as_float(v[j + 5]) * sg);
            u.w = pack_bf16x2(__uint_as_float(v[j + 6]) * sg, __uint_as_float(v[j + 7]) * sg);
            st_global_v4_hint(o + j, u, pol_out);
          }
        }
      };
      // The warp's four chunks are read two at a time (one wait per pair). The
      // slice shared with the other accumulator (chunks 6,7 of buffer 0,
      // chunks 0,1 of buffer 1) belongs to one warp of each lane quarter: it
      // reads that pair first and releases the MMA before any arithmetic; the
      // other warps release at once.
      const bool owns_shared = buf ? half == 0 : half == 1;
      if (!owns_shared) release();
      const int i0 = buf ? 0 : 2;   // first pair (of the warp's chunks half * 4 + i)
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const int c = half * 4 + (pr == 0 ? i0 : 2 - i0);
        uint32_t v0[32], v1[32];
        tmem_ld_32x32b_x32(acc + c * 32, v0);
        tmem_ld_32x32b_x32(acc + (c + 1) * 32, v1);
        tmem_ld_wait();
        if (pr == 0 && owns_shared) release();
        emit(c, v0);
        emit(c + 1, v1);
      }
      ++local;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace lmoe
