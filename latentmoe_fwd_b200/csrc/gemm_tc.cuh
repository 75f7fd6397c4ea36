// Persistent BF16 tensor-core GEMM for sm_100a (tcgen05 + TMEM + TMA).
//
//   D[rows, cols] = A[rows, K] . B[cols, K]^T   (both operands K-major)
//
// One CTA per SM loops over output tiles. Warp roles:
//   warp 0      TMA producer: streams 64-wide K slices of A and B into a ring
//               of shared-memory stages (128-byte swizzle).
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN,
//               K=16 each) into one of two TMEM accumulators, and commits
//               stage releases / accumulator-ready signals to mbarriers.
//   warps 2..5  epilogue: tcgen05.ld the accumulator (one TMEM lane = one row
//               per thread), apply the fused epilogue, store to global.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile i+1.
//
// Tile kinds:
//   normal: A = activation rows (128 per tile), B = weight rows (BN per tile);
//           dense GEMMs only.
//   swap:   A = weight rows (128 per tile), B = activation rows (<= BN tokens);
//           used when the token count is tiny and the GEMM streams weights.
//   grouped (swap only): activation rows are the expert-grouped padded buffer;
//           the weight operand is a 3-D map [experts][rows][K] indexed by the
//           tile's expert.
// Up to two K segments are summed into one accumulator (used for
// out = c W_up^T + sum_s as_s Ws2_s^T).
#pragma once

#include "lmoe_device.cuh"

namespace lmoe {

enum EpiKind : int {
  EPI_F32_BIAS = 0,   // out f32 = acc (+ bias[col])
  EPI_BF16 = 1,       // out bf16 = acc
  EPI_SQRELU = 2,     // out bf16 = relu(acc)^2
  EPI_GATE = 3,       // out bf16 = acc * row_scale[row]
  EPI_ADD_RES = 4,    // out bf16 = acc + residual[row][col]
  EPI_PARTIAL = 5,    // split-K: fp32 partial sums, the epilogue runs in the reduction
  EPI_SQRELU_Q8 = 7,  // out E4M3 byte = E4M3(relu(acc * s_a * s_w)^2 / out_scale)
  EPI_SCALE = 8       // out bf16 = acc * s_a * s_w
};

struct TcSeg {
  int kblocks;     // 64-wide K blocks in this segment
  int a_kgroup;    // >0: the K axis of A is split into groups of a_kgroup along its 3rd dim
  int b_kgroup;    // same for B
};

struct TcParams {
  int swap;        // 0 normal, 1 swap (A = weights)
  int grouped;     // 1: expert-grouped activations
  int rows;        // dense: activation rows (tokens)
  int cols;        // output features (weight rows per expert)
  int nseg;        // 1 or 2
  TcSeg seg[2];
  const int* offsets;         // grouped: [G+1] valid-row offsets
  const int* padded_offsets;  // grouped: [G+1] padded-row offsets (multiples of 128)
  int groups;                 // grouped: number of experts
  void* out;
  long long ld_out;           // elements
  const float* bias;          // EPI_F32_BIAS: [cols] or nullptr
  const float* row_scale;     // EPI_GATE: per activation row, or nullptr (= 1)
  const __nv_bfloat16* residual;
  long long ld_res;
  int ksplit;                 // >1: split the K blocks of every tile; partial sums go to `partial`
  float* partial;             // [ksplit][rows][cols] fp32 (split-K only)
  // FP8 operands (E4M3 codes, 1 byte each; K blocks of 128 elements, the same
  // 128 bytes per row per stage as BF16): tcgen05.mma kind::f8f6f4
  int fp8;
  const float* scale_a;       // EPI_SQRELU_Q8 / EPI_SCALE: per-tensor scales of the two operands
  const float* scale_w;       //   (device scalars; the product multiplies the accumulator)
  const float* out_scale;     // EPI_SQRELU_Q8: static scale of the E4M3 output
  // CTA-pair grouped launches only: one dense problem computed in the same
  // launch, out_x[rows_x, cols_x] = epi(X[rows_x, K_x] . Wx[cols_x, K_x]^T)
  int rows_x;                 // 0: none
  int cols_x;
  int kblocks_x;
  int kgroup_x;               // >0: the extra weights are [K / kgroup_x][cols_x][kgroup_x] (K split in groups)
  void* out_x;
  long long ld_out_x;
  DevErr err;
};

template <int BN, int STAGES>
struct TcSmem {
  static constexpr int kABytes = 128 * 128;           // 128 rows x 64 bf16
  static constexpr int kBBytes = BN * 128;            // BN rows x 64 bf16
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  // full[STAGES], empty[STAGES], tfull[2], tempty[2], drain, tmem ptr, abort
  static constexpr int kPrefixOffset = kBarOffset + (2 * STAGES + 5) * 8 + 16;
  // weight-major grouped tiles: prefix over experts of their tile counts
  static constexpr int kMaxGroups = 1024;
  // weight-major epilogue: one 32 x 32 BF16 transpose tile per epilogue warp
  static constexpr int kEpiOffset = (kPrefixOffset + (kMaxGroups + 1) * 4 + 15) / 16 * 16;
  // per epilogue warp: a 32 x 32 BF16 transpose tile (80-byte row pitch, bank-conflict free)
  static constexpr int kEpiWarpBytes = 32 * 80;
  static constexpr int kBytes = kEpiOffset + 4 * kEpiWarpBytes + 1024;  // +1024 alignment slack
};

struct TileInfo {
  int valid;      // 0: skip (empty expert)
  int expert;     // grouped: expert; else 0
  int act0;       // first activation row of the tile
  int act_n;      // valid activation rows (<= 128 normal, <= BN swap)
  int w0;         // first weight row (output feature) of the tile
  int split;      // split-K index
  int kb0, kb1;   // K blocks [kb0, kb1) of this tile
  int wshared;    // weight-major: other tiles of this expert read the same weight rows
};

// Weight-major grouped tiles: expert e owns ceil(n_e / BN) token tiles times
// ceil(cols / 128) weight tiles. prefix[e] = tiles of experts before e, built
// by every CTA in shared memory at start.
template <int BN>
__device__ __forceinline__ void build_tile_prefix(const TcParams& p, int* prefix) {
  const int ntw = (p.cols + 127) / 128;
  for (int e = threadIdx.x; e < p.groups; e += blockDim.x) {
    int n_e = __ldg(p.offsets + e + 1) - __ldg(p.offsets + e);
    if (kChecks) {   // the expert's rows must fit its padded range inside the buffer
      const int ps = __ldg(p.padded_offsets + e), pe = __ldg(p.padded_offsets + e + 1);
      if (n_e < 0 || ps < 0 || pe > p.rows || ps + n_e > pe) {
        dev_report(p.err, kErrBounds, 0x5100);
        n_e = 0;
      }
    }
    prefix[e + 1] = ((n_e + BN - 1) / BN) * ntw;
  }
  if (threadIdx.x == 0) prefix[0] = 0;
  __syncthreads();
  if (threadIdx.x < 32) {   // inclusive scan of prefix[1..groups] by one warp
    const int lane = threadIdx.x;
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

template <int BN>
__device__ __forceinline__ int tc_num_tiles(const TcParams& p, const int* prefix) {
  const int ntw_normal = (p.cols + BN - 1) / BN;
  const int ntw_swap = (p.cols + 127) / 128;
  int n;
  if (!p.swap) {
    n = ((p.rows + 127) / 128) * ntw_normal;
  } else {
    n = p.grouped ? prefix[p.groups] : ntw_swap;
  }
  return n * p.ksplit;
}

template <int BN>
__device__ __forceinline__ TileInfo tc_tile(const TcParams& p, int t, int kb_total, const int* prefix) {
  TileInfo ti;
  ti.valid = 1;
  ti.expert = 0;
  ti.wshared = 0;
  ti.split = t % p.ksplit;
  t /= p.ksplit;
  {
    const int per = (kb_total + p.ksplit - 1) / p.ksplit;
    ti.kb0 = ti.split * per;
    ti.kb1 = min(kb_total, ti.kb0 + per);
    if (ti.kb0 >= ti.kb1) ti.valid = 0;
  }
  if (!p.swap) {
    const int ntw = (p.cols + BN - 1) / BN;
    const int nt = t % ntw, mt = t / ntw;
    ti.w0 = nt * BN;
    ti.act0 = mt * 128;
    ti.act_n = min(128, p.rows - ti.act0);
  } else {
    const int ntw = (p.cols + 127) / 128;
    if (p.grouped) {
      // largest e with prefix[e] <= t (it owns at least one tile)
      int lo = 0, hi = p.groups - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
      }
      const int e = lo;
      const int n_e = __ldg(p.offsets + e + 1) - __ldg(p.offsets + e);
      const int ntt = (n_e + BN - 1) / BN;
      const int local = t - prefix[e];
      // the weight tiles of one token tile are consecutive: CTAs running at the
      // same time share the token rows, and the expert's weights (reused by
      // every token tile) stay in L2
      const int tt = local / ntw, mw = local % ntw;
      ti.expert = e;
      ti.wshared = ntt > 1;
      ti.w0 = mw * 128;
      ti.act0 = __ldg(p.padded_offsets + e) + tt * BN;
      ti.act_n = min(BN, n_e - tt * BN);
      if (ti.act_n <= 0) ti.valid = 0;
    } else {
      ti.w0 = (t % ntw) * 128;
      ti.act0 = 0;
      ti.act_n = min(p.rows, BN);
    }
  }
  return ti;
}

// MMA N of a tile: its rows (normal) or its tokens rounded up to 16 (weight-major).
template <int BN>
__device__ __forceinline__ int tile_mma_n(const TcParams& p, const TileInfo& ti) {
  if (!p.swap) return BN;
  const int n = (ti.act_n + 15) & ~15;
  return n < 16 ? 16 : n;
}

// Product of the two operands' FP8 scales (1 for BF16 operands).
__device__ __forceinline__ float fp8_acc_scale(const TcParams& p) {
  return (p.scale_a && p.scale_w) ? __fmul_rn(__ldg(p.scale_a), __ldg(p.scale_w)) : 1.0f;
}

// E4M3 code of relu(acc * sc)^2 / out_scale (round to nearest even, saturating).
__device__ __forceinline__ uint32_t sqrelu_e4m3(float acc, float sc, float out_scale) {
  const float h = fmaxf(__fmul_rn(acc, sc), 0.0f);
  return cvt_to_e4m3(__fdiv_rn(__fmul_rn(h, h), out_scale));
}

template <int EPI>
__device__ __forceinline__ float epi_value(float acc, const TcParams& p, long long row, int col) {
  if (EPI == EPI_SCALE) {
    return __fmul_rn(acc, fp8_acc_scale(p));
  } else if (EPI == EPI_SQRELU) {
    float r = fmaxf(acc, 0.0f);
    return r * r;
  } else if (EPI == EPI_GATE) {
    return p.row_scale ? acc * __ldg(p.row_scale + row) : acc;
  } else if (EPI == EPI_F32_BIAS) {
    return p.bias ? acc + __ldg(p.bias + col) : acc;
  } else if (EPI == EPI_ADD_RES) {
    return acc + __bfloat162float(p.residual[row * p.ld_res + col]);
  }
  return acc;
}

template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(192, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ CUtensorMap tmBs, const TcParams p) {
  pdl_begin();
  using S = TcSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_ptr + 1);
  int* tile_prefix = reinterpret_cast<int*>(smem + S::kPrefixOffset);
  __nv_bfloat16* epi_tile = reinterpret_cast<__nv_bfloat16*>(smem + S::kEpiOffset);

  const int warp = warp_id();
  const int lane = lane_id();
  if (p.swap && p.grouped) build_tile_prefix<BN>(p, tile_prefix);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB0);
    if (p.nseg > 1) {
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB1);
    }
  }
  if (warp == 1) tmem_alloc(tmem_ptr, S::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_ptr;

  const int ntiles = tc_num_tiles<BN>(p, tile_prefix);
  const int kb_total = p.seg[0].kblocks + (p.nseg > 1 ? p.seg[1].kblocks : 0);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      const uint64_t pol_w = policy_evict_first();   // weights: streamed
      const uint64_t pol_a = policy_evict_last();    // activations: reused across tiles
      const uint64_t pol_n = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0;
      uint32_t last_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const TileInfo ti = tc_tile<BN>(p, t, kb_total, tile_prefix);
        if (!ti.valid) continue;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, 0x100 + stage)) { ok = false; break; }
          uint8_t* sa = smem + stage * S::kStageBytes;
          uint8_t* sb = sa + S::kABytes;
          // weight-major tiles of at most 32 tokens fetch a 32-row token box
          const bool small_b = BN > 32 && p.swap && p.grouped && ti.act_n <= 32;
          mbar_arrive_expect_tx(&full[stage], small_b ? S::kABytes + 32 * 128 : S::kStageBytes);
          const int sg = (p.nseg > 1 && kb >= p.seg[0].kblocks) ? 1 : 0;
          const int k = (sg ? kb - p.seg[0].kblocks : kb) * (p.fp8 ? 128 : 64);
          const CUtensorMap* ma = sg ? &tmA1 : &tmA0;
          const CUtensorMap* mb = sg ? &tmB1 : &tmB0;
          const int akg = p.seg[sg].a_kgroup, bkg = p.seg[sg].b_kgroup;
          int a_row, a_grp, b_row, b_grp;
          if (!p.swap) {
            a_row = ti.act0; a_grp = 0; b_row = ti.w0; b_grp = ti.expert;
          } else {
            a_row = ti.w0; a_grp = ti.expert; b_row = ti.act0; b_grp = 0;
          }
          // L2 policy per operand:
          //  * dense token-major tiles (the projections and the router at large
          //    T): every row block reads all of the weight matrix, while a row
          //    block of activations is read only by the tiles next to it in the
          //    tile order, which run at the same time: weights kept (evict
          //    last), activations normal, so a long activation stream cannot
          //    push the weights out;
          //  * grouped token-major tiles: an expert's weights serve only its
          //    own row blocks: weights streamed, activations kept;
          //  * weight-major tiles: weights kept when other token tiles of the
          //    expert read them again, streamed otherwise; activations kept.
          const bool dense_tm = !p.swap && !p.grouped;
          const uint64_t pa = p.swap ? (ti.wshared ? pol_a : pol_w) : (dense_tm ? pol_n : pol_a);
          const uint64_t pb = p.swap ? (ti.wshared ? pol_n : pol_a) : (dense_tm ? pol_a : pol_w);
          if (akg > 0) tma_load_3d(sa, ma, &full[stage], k % akg, a_row, k / akg, pa);
          else tma_load_3d(sa, ma, &full[stage], k, a_row, a_grp, pa);
          if (bkg > 0) tma_load_3d(sb, mb, &full[stage], k % bkg, b_row, k / bkg, pb);
          else if (small_b) tma_load_3d(sb, &tmBs, &full[stage], k, b_row, b_grp, pb);
          else tma_load_3d(sb, mb, &full[stage], k, b_row, b_grp, pb);
          issued_mask |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (*abort_flag) {
        // let every load already issued land before the CTA's memory goes away
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s)) {
            long long t0 = clock64();
            while (!mbar_try_wait(&full[s], (last_par >> s) & 1) && clock64() - t0 < kWaitLimitCycles / 4) {}
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------

      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      bool any = false;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const TileInfo ti = tc_tile<BN>(p, t, kb_total, tile_prefix);
        if (!ti.valid) continue;
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err, 0x200 + acc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        const uint32_t idesc = p.fp8 ? idesc_e4m3_f32(128, tile_mma_n<BN>(p, ti))
                                     : idesc_bf16_f32(128, tile_mma_n<BN>(p, ti));
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, 0x300 + stage)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * S::kStageBytes);
          const uint32_t sb = sa + S::kABytes;
          if (p.fp8) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_e4m3(d_tmem, sdesc_kmajor_sw128(sa + kk * 32), sdesc_kmajor_sw128(sb + kk * 32), idesc,
                       (kb != ti.kb0 || kk != 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(d_tmem, sdesc_kmajor_sw128(sa + kk * 32), sdesc_kmajor_sw128(sb + kk * 32), idesc,
                       (kb != ti.kb0 || kk != 0) ? 1u : 0u);
          }
          any = true;
          mma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        ++local;
      }
      if (any) {
        mma_commit(drain);
        long long t0 = clock64();
        while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitLimitCycles / 4) {}
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;          // TMEM lane quadrant this warp may access
    const int r = q * 32 + lane;     // accumulator row of this thread
    int local = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      const TileInfo ti = tc_tile<BN>(p, t, kb_total, tile_prefix);
      if (!ti.valid) continue;
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, 0x400 + acc)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
      const int nchunks = p.swap ? (ti.act_n + 31) / 32 : BN / 32;
#pragma unroll 1
      for (int c = 0; c < nchunks; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_row + c * 32, v);
        tmem_ld_wait();
        if (!p.swap) {
          const long long row = ti.act0 + r;
          if (r < ti.act_n) {
            const int col0 = ti.w0 + c * 32;
            if (EPI == EPI_PARTIAL) {
              float* o = p.partial + (static_cast<long long>(ti.split) * p.rows + row) * p.cols + col0;
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                if (col0 + j < p.cols)
                  *reinterpret_cast<float4*>(o + j) = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                                                   __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
            } else if (EPI == EPI_SQRELU_Q8) {
              const float sc = fp8_acc_scale(p);
              const float os = __ldg(p.out_scale);
              uint32_t w[8];
#pragma unroll
              for (int j = 0; j < 8; ++j)
                w[j] = sqrelu_e4m3(__uint_as_float(v[4 * j]), sc, os) |
                       (sqrelu_e4m3(__uint_as_float(v[4 * j + 1]), sc, os) << 8) |
                       (sqrelu_e4m3(__uint_as_float(v[4 * j + 2]), sc, os) << 16) |
                       (sqrelu_e4m3(__uint_as_float(v[4 * j + 3]), sc, os) << 24);
              uint8_t* o = reinterpret_cast<uint8_t*>(p.out) + row * p.ld_out + col0;
              if (col0 + 16 <= p.cols) *reinterpret_cast<uint4*>(o) = make_uint4(w[0], w[1], w[2], w[3]);
              if (col0 + 32 <= p.cols) *reinterpret_cast<uint4*>(o + 16) = make_uint4(w[4], w[5], w[6], w[7]);
            } else if (EPI == EPI_F32_BIAS) {
              float* o = reinterpret_cast<float*>(p.out) + row * p.ld_out + col0;
#pragma unroll
              for (int j = 0; j < 32; j += 4) {
                if (col0 + j < p.cols) {
                  float4 f;
                  f.x = epi_value<EPI>(__uint_as_float(v[j + 0]), p, row, col0 + j + 0);
                  f.y = epi_value<EPI>(__uint_as_float(v[j + 1]), p, row, col0 + j + 1);
                  f.z = epi_value<EPI>(__uint_as_float(v[j + 2]), p, row, col0 + j + 2);
                  f.w = epi_value<EPI>(__uint_as_float(v[j + 3]), p, row, col0 + j + 3);
                  *reinterpret_cast<float4*>(o + j) = f;
                }
              }
            } else {
              __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + row * p.ld_out + col0;
#pragma unroll
              for (int j = 0; j < 32; j += 8) {
                if (col0 + j < p.cols) {
                  uint4 u;
                  u.x = pack_bf16x2(epi_value<EPI>(__uint_as_float(v[j + 0]), p, row, col0 + j + 0),
                                    epi_value<EPI>(__uint_as_float(v[j + 1]), p, row, col0 + j + 1));
                  u.y = pack_bf16x2(epi_value<EPI>(__uint_as_float(v[j + 2]), p, row, col0 + j + 2),
                                    epi_value<EPI>(__uint_as_float(v[j + 3]), p, row, col0 + j + 3));
                  u.z = pack_bf16x2(epi_value<EPI>(__uint_as_float(v[j + 4]), p, row, col0 + j + 4),
                                    epi_value<EPI>(__uint_as_float(v[j + 5]), p, row, col0 + j + 5));
                  u.w = pack_bf16x2(epi_value<EPI>(__uint_as_float(v[j + 6]), p, row, col0 + j + 6),
                                    epi_value<EPI>(__uint_as_float(v[j + 7]), p, row, col0 + j + 7));
                  *reinterpret_cast<uint4*>(o + j) = u;
                }
              }
            }
          }
        } else if (EPI != EPI_PARTIAL && EPI != EPI_F32_BIAS && EPI != EPI_SQRELU_Q8) {
          // weight-major, BF16 out: this lane owns output feature w0 + r and 32
          // tokens; transpose the warp's 32 x 32 block through shared memory so
          // each token's 32 features go out as 16-byte stores
          __nv_bfloat16* tb = epi_tile + (warp & 3) * (S::kEpiWarpBytes / 2);
          const int col = ti.w0 + r;
          // per-token operands of the chunk are fetched before any store: the
          // gate of token c*32+lane by this lane (one coalesced load, then
          // shuffles), the residual row values into registers
          float gate = 1.0f;
          if (EPI == EPI_GATE && p.row_scale) {
            const int tk = c * 32 + lane;
            gate = tk < ti.act_n ? __ldg(p.row_scale + ti.act0 + tk) : 0.0f;
          }
          float res[32];
          if (EPI == EPI_ADD_RES) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const bool live = c * 32 + j < ti.act_n && col < p.cols;
              res[j] = live ? __bfloat162float(p.residual[(ti.act0 + c * 32 + j) * p.ld_res + col]) : 0.0f;
            }
          }
          const float fp8_sc = EPI == EPI_SCALE ? fp8_acc_scale(p) : 1.0f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float val = __uint_as_float(v[j]);
            if (EPI == EPI_SQRELU) {
              val = fmaxf(val, 0.0f);
              val = val * val;
            } else if (EPI == EPI_GATE) {
              val = val * __shfl_sync(0xffffffffu, gate, j);
            } else if (EPI == EPI_ADD_RES) {
              val = val + res[j];
            } else if (EPI == EPI_SCALE) {
              val = __fmul_rn(val, fp8_sc);
            }
            tb[j * 32 + lane] = __float2bfloat16_rn(val);
          }
          __syncwarp();
          const int seg = lane & 3;              // 8 features of the warp's 32
          const int col0 = ti.w0 + q * 32 + seg * 8;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int j = (lane >> 2) + 8 * i;   // token within the chunk
            const int tok = c * 32 + j;
            if (tok < ti.act_n && col0 < p.cols) {
              const uint4 u = *reinterpret_cast<const uint4*>(tb + j * 32 + seg * 8);
              __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out) + (ti.act0 + tok) * p.ld_out + col0;
              *reinterpret_cast<uint4*>(o) = u;
            }
          }
          __syncwarp();
        } else {
          // weight-major, fp32 or split-K partial out: scalar stores
          const int col = ti.w0 + r;
          if (col < p.cols) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int tok = c * 32 + j;
              if (tok < ti.act_n) {
                const long long row = ti.act0 + tok;
                if (EPI == EPI_PARTIAL) {
                  p.partial[(static_cast<long long>(ti.split) * p.rows + row) * p.cols + col] = __uint_as_float(v[j]);
                  continue;
                }
                if (EPI == EPI_SQRELU_Q8) {
                  reinterpret_cast<uint8_t*>(p.out)[row * p.ld_out + col] = static_cast<uint8_t>(
                      sqrelu_e4m3(__uint_as_float(v[j]), fp8_acc_scale(p), __ldg(p.out_scale)));
                  continue;
                }
                const float val = epi_value<EPI>(__uint_as_float(v[j]), p, row, col);
                if (EPI == EPI_F32_BIAS)
                  reinterpret_cast<float*>(p.out)[row * p.ld_out + col] = val;
                else
                  reinterpret_cast<__nv_bfloat16*>(p.out)[row * p.ld_out + col] = __float2bfloat16_rn(val);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      ++local;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

// Split-K reduction: out[row, col] = epi(sum over splits in order of partial[s][row][col]).
template <int EPI>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const TcParams p) {
  pdl_begin();
  const long long n = static_cast<long long>(p.rows) * p.cols;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float acc = 0.0f;
    for (int sp = 0; sp < p.ksplit; ++sp) acc += p.partial[sp * n + i];
    const long long row = i / p.cols;
    const int col = static_cast<int>(i % p.cols);
    if (EPI == EPI_SQRELU_Q8) {
      reinterpret_cast<uint8_t*>(p.out)[row * p.ld_out + col] =
          static_cast<uint8_t>(sqrelu_e4m3(acc, fp8_acc_scale(p), __ldg(p.out_scale)));
      continue;
    }
    const float val = epi_value<EPI>(acc, p, row, col);
    if (EPI == EPI_F32_BIAS)
      reinterpret_cast<float*>(p.out)[row * p.ld_out + col] = val;
    else
      reinterpret_cast<__nv_bfloat16*>(p.out)[row * p.ld_out + col] = __float2bfloat16_rn(val);
  }
}

}  // namespace lmoe
