// NVFP4 training-recipe quantiser: the operands of the expert GEMMs' dgrad
// and wgrad (greeksharifa page on the Nemotron 3 whitepaper, section 2.4
// "NVFP4 Training"; notes.yuuk.io page, section 4 "NVFP4 pre-training"):
// gradients are rounded stochastically, the wgrad inputs get a random
// Hadamard transform along the contraction (token) dimension, weights use
// 16 x 16 scale blocks. One kernel covers every combination the recipe uses:
//
//   out = in or in^T (LMOE_QX_TRANSPOSE: blocks run along the input's rows)
//   each 16-block v of out's rows -> H16 diag(s) v / 4 (LMOE_QX_RHT)
//   two-level NVFP4 scales as lmoe_nvfp4_quantize (1 x 16, or 16 x 16 blocks)
//   elements rounded to nearest even, or stochastically (LMOE_QX_SR) with
//   uniforms from Philox-4x32-10 at the element's index in `out`.
//
// Arithmetic: the transform is formed in fp64 (exact for BF16 inputs), and
// every step after it is an IEEE fp64 operation rounded to fp32 where the
// recipe's step is an fp32 one, so the codes equal those of the same steps
// taken in fp64 and rounded, input for input.
#include <cuda_bf16.h>

#include "lmoe_device.cuh"
#include "lmoe_internal.h"

namespace lmoe {
namespace {

constexpr int kXThreads = 256;

// E4M3 code -> exact value: subnormal f * 2^-9, normal (8 + f) * 2^(e - 10).
__device__ __forceinline__ double e4m3_exact(uint32_t c) {
  const int e = (c >> 3) & 15, f = c & 7;
  // f * 2^-9 or (8 + f) * 2^(e - 10): a small integer times a power of two
  // built from its exponent bits (both exact)
  const int ex = e == 0 ? -9 : e - 10;
  return static_cast<double>(e == 0 ? f : 8 + f) * __longlong_as_double(static_cast<long long>(ex + 1023) << 52);
}

// Philox-4x32-10 (Salmon et al., "Parallel random numbers: as easy as 1, 2, 3",
// SC11): ten rounds; each takes the 64-bit products of words 0 and 2 with the
// multipliers 0xD2511F53 and 0xCD9E8D57, and the key grows by the Weyl
// constants 0x9E3779B9 and 0xBB67AE85 between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// 16 uniforms of elements i0 .. i0+15 (i0 a multiple of 4): element i takes
// word i % 4 of Philox at counter (i / 4 low word, i / 4 high word, stream, 0)
// under key (seed low word, seed high word); u = (word >> 8) * 2^-24.
__device__ __forceinline__ void sr_uniforms16(uint64_t i0, uint64_t seed, uint32_t stream, float (&u)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint64_t c = (i0 >> 2) + q;
    const uint4 w = philox4x32_10(make_uint4(static_cast<uint32_t>(c), static_cast<uint32_t>(c >> 32), stream, 0u),
                                  static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
    constexpr float k2m24 = 1.0f / 16777216.0f;   // 2^-24: the products are exact
    u[4 * q + 0] = static_cast<float>(w.x >> 8) * k2m24;
    u[4 * q + 1] = static_cast<float>(w.y >> 8) * k2m24;
    u[4 * q + 2] = static_cast<float>(w.z >> 8) * k2m24;
    u[4 * q + 3] = static_cast<float>(w.w >> 8) * k2m24;
  }
}

struct QxParams {
  const void* in;
  int bf16;              // input BF16 (else F32)
  int64_t rows, cols;    // input dims
  int transpose;
  int rht;
  uint32_t signs;        // RHT: bit i set = sign -1 on element i of a block
  int sr;
  uint64_t seed;
  uint32_t stream;
  int block2d;
  int tiled;
  const float* global_in;
  const double* partials;
  int np;
  uint8_t* codes;
  uint8_t* sf;
  float* global_out;
  int64_t pitch;         // elements per stored output row (>= out cols; the rest stored as zero codes and scales)
  // grouped launches (gridDim.y groups, one matrix each, with its own global
  // scale): strides between the groups' inputs (elements), codes and scales (bytes)
  int64_t gs_in, gs_codes, gs_sf;
  // ragged groups instead (gtab non-null): per group {first input row, input
  // rows, codes offset, scales offset (bytes), output pitch (0: out cols),
  // rows holding data}; group g draws its SR uniforms on stream + g * stream_step
  const int64_t* gtab;
  uint32_t stream_step;
  int vec;               // input 16-byte aligned: row segments read with 16-byte loads
  int64_t ld;            // elements per destination row (codes, and tiled scale atoms); 0: pitch
};

// The parameters of group blockIdx.y: its input, outputs, global scale and
// amax partials.
__device__ __forceinline__ QxParams qx_group(const QxParams& p0) {
  QxParams p = p0;
  const int64_t g = blockIdx.y;
  if (p0.gtab) {
    const int64_t* t = p0.gtab + g * 6;
    p.in = static_cast<const uint8_t*>(p0.in) + t[0] * p0.cols * (p0.bf16 ? 2 : 4);
    p.rows = t[1];
    p.codes += t[2];
    p.sf += t[3];
    p.pitch = t[4] > 0 ? t[4] : (p0.transpose ? t[1] : p0.cols);
    p.stream = p0.stream + static_cast<uint32_t>(g) * p0.stream_step;
    if (p.global_out) p.global_out += g;
    if (p.partials) p.partials += g * p0.np;
  } else if (g) {
    p.in = static_cast<const uint8_t*>(p0.in) + g * p0.gs_in * (p0.bf16 ? 2 : 4);
    p.codes += g * p0.gs_codes;
    p.sf += g * p0.gs_sf;
    if (p.global_out) p.global_out += g;
    if (p.partials) p.partials += g * p0.np;
  }
  return p;
}

__device__ __forceinline__ double load_in(const QxParams& p, int64_t r, int64_t c) {
  if (p.bf16) return static_cast<double>(__bfloat162float(static_cast<const __nv_bfloat16*>(p.in)[r * p.cols + c]));
  return static_cast<double>(static_cast<const float*>(p.in)[r * p.cols + c]);
}

// The 16 values of output row ro, block j (transformed when asked).
__device__ __forceinline__ void load_block(const QxParams& p, int64_t ro, int64_t j, double (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = p.transpose ? load_in(p, j * 16 + i, ro) : load_in(p, ro, j * 16 + i);
  if (p.rht) {
    // H16 diag(s) v / 4: signs, then the fast Walsh-Hadamard butterflies
    // (Sylvester order), then the exact division by 4
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if ((p.signs >> i) & 1u) v[i] = -v[i];
#pragma unroll
    for (int h = 1; h < 16; h <<= 1)
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if ((i & h) == 0) {
          const double a = v[i], b = v[i + h];
          v[i] = a + b;
          v[i + h] = a - b;
        }
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] *= 0.25;
  }
}

// Without the transform every value is an fp32 number, and so is each step
// below (fp32 IEEE division gives the correctly rounded quotient, which the
// fp64 quotient rounded to fp32 equals: 53 >= 2 * 24 + 2 bits), so this path
// takes the same decisions in fp32.
__device__ __forceinline__ void load_block_f32(const QxParams& p, int64_t ro, int64_t j, float (&v)[16]) {
  if (!p.transpose && p.vec) {
    if (p.bf16) {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.in) + ro * p.cols + j * 16);
      const uint4 a = __ldg(src), b = __ldg(src + 1);
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    } else {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(p.in) + ro * p.cols + j * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 f = __ldg(src + i);
        v[4 * i] = f.x;
        v[4 * i + 1] = f.y;
        v[4 * i + 2] = f.z;
        v[4 * i + 3] = f.w;
      }
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int64_t r = p.transpose ? j * 16 + i : ro, c = p.transpose ? ro : j * 16 + i;
    v[i] = p.bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p.in)[r * p.cols + c])
                  : static_cast<const float*>(p.in)[r * p.cols + c];
  }
}

// E4M3 code -> value in fp32 (exact: at most 4 significant bits, a normal
// power of two between 2^-9 and 2^5).
__device__ __forceinline__ float e4m3_exact_f(uint32_t c) {
  const int e = (c >> 3) & 15, f = c & 7;
  const int ex = e == 0 ? -9 : e - 10;
  return static_cast<float>(e == 0 ? f : 8 + f) * __int_as_float((ex + 127) << 23);
}

__device__ __forceinline__ int64_t out_rows(const QxParams& p) { return p.transpose ? p.cols : p.rows; }
__device__ __forceinline__ int64_t out_cols(const QxParams& p) { return p.transpose ? p.rows : p.cols; }

// Pass 1: per-CTA maxima of |out| (fp64, exact).
template <bool RHT>
__global__ void __launch_bounds__(kXThreads, RHT ? 4 : 6) qx_amax_kernel(const QxParams p0,
                                                                       double* __restrict__ partials) {
  pdl_begin();
  const QxParams p = qx_group(p0);
  partials += static_cast<int64_t>(blockIdx.y) * gridDim.x;
  __shared__ double red[kXThreads / 32];
  const int64_t nb = out_cols(p) / 16, total = out_rows(p) * nb;
  double m = 0.0;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < total;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    // transposed input: consecutive threads take consecutive output rows
    // (consecutive input columns) of one block column, so loads coalesce
    const int64_t ro = p.transpose ? b % out_rows(p) : b / nb;
    const int64_t j = p.transpose ? b / out_rows(p) : b % nb;
    if constexpr (RHT) {
      double v[16];
      load_block(p, ro, j, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) m = fmax(m, fabs(v[i]));
    } else {
      float v[16];
      load_block_f32(p, ro, j, v);
      float mf = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) mf = fmaxf(mf, fabsf(v[i]));
      m = fmax(m, static_cast<double>(mf));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    double r = 0.0;
    for (int i = 0; i < kXThreads / 32; ++i) r = fmax(r, red[i]);
    partials[blockIdx.x] = r;
  }
}

// Stochastic E2M1 code of v (fp32 value): |v| >= 6 -> 6; else, between grid
// neighbours lo <= |v| < hi, hi when u * (hi - lo) < |v| - lo, else lo; the
// sign bit is the sign of v. Both sides are exact in fp32: hi - lo is a power
// of two, u has 24 bits, and lo <= |v| < hi <= 2 lo (or lo = 0) makes the
// difference exact. The grid (0, 0.5, 1, 1.5, 2, 3, 4, 6) is walked with
// compares and selects, so nothing is indexed at run time.
__device__ __forceinline__ uint32_t e2m1_sr(float v, float u) {
  const float a = fabsf(v);
  uint32_t lo = 0;
  float l = 0.0f, h = 0.5f;
  if (a >= 0.5f) { lo = 1; l = 0.5f; h = 1.0f; }
  if (a >= 1.0f) { lo = 2; l = 1.0f; h = 1.5f; }
  if (a >= 1.5f) { lo = 3; l = 1.5f; h = 2.0f; }
  if (a >= 2.0f) { lo = 4; l = 2.0f; h = 3.0f; }
  if (a >= 3.0f) { lo = 5; l = 3.0f; h = 4.0f; }
  if (a >= 4.0f) { lo = 6; l = 4.0f; h = 6.0f; }
  uint32_t code = lo;
  if (a >= 6.0f) code = 7;
  else if (__fmul_rn(u, h - l) < __fsub_rn(a, l)) code = lo + 1;
  return code | (signbit(v) ? 8u : 0u);
}

__device__ __forceinline__ int64_t tiled_off(int64_t row, int64_t j, int64_t groups64) {
  return ((row >> 7) * groups64 + (j >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (j & 3);
}

// Pass 2: a thread per output row and 16-column block; the 16 rows of a
// 16-row group sit in one half-warp (lane & 15 = row in the group), so a
// 16 x 16 block's amax is a half-warp reduction. The item count is rounded up
// to whole warps; items past the end take part in the reductions only.
// Latency-bound: occupancy matters more than registers (bounded to 4 CTAs per
// SM, 3 for the transform path, at no or negligible spilling).
template <bool RHT>
__global__ void __launch_bounds__(kXThreads, RHT ? 3 : 4) qx_encode_kernel(const QxParams p0) {
  pdl_begin();
  const QxParams p = qx_group(p0);
  __shared__ double red[kXThreads / 32];
  __shared__ float s_gs;
  // global scale: s_g = fp32(amax / 2688) from the fp64 amax (1 when 0)
  if (p.global_in) {
    if (threadIdx.x == 0) s_gs = __ldg(p.global_in);
  } else {
    double m = 0.0;
    for (int i = threadIdx.x; i < p.np; i += blockDim.x) m = fmax(m, p.partials[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      double r = 0.0;
      for (int i = 0; i < kXThreads / 32; ++i) r = fmax(r, red[i]);
      s_gs = r == 0.0 ? 1.0f : __double2float_rn(r / 2688.0);
    }
  }
  __syncthreads();
  const float s_g = s_gs;
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.global_out) *p.global_out = s_g;
  const float t = __fmul_rn(s_g, 6.0f);
  const int64_t R = out_rows(p), C = out_cols(p), nb = C / 16;
  const int64_t nb_store = p.pitch / 16;   // stored blocks per row; those past nb are zero
  const int64_t groups64 = (p.pitch + 63) / 64;
  const int64_t ld = p.ld > 0 ? p.ld : p.pitch;
  const int64_t ld64 = (ld + 63) / 64;
  const int64_t rg_cov = p.tiled ? (R + 127) / 128 * 8 : (R + 15) / 16;   // 16-row groups, tiled padding
  const int64_t nb_cov = p.tiled ? groups64 * 4 : nb_store;
  const int64_t items = rg_cov * nb_cov * 16;
  const int64_t items32 = (items + 31) / 32 * 32;
  const int i16 = threadIdx.x & 15;
  // One item per thread and pass: output row ro, block j. `fetch` reads its 16
  // values and their amax; `finish` forms the 16 x 16 amax (half-warp
  // shuffles, every lane takes part), then encodes and stores. (Two items in
  // flight per thread measured slower: the extra registers cost occupancy.)
  struct Item {
    bool live, has;
    int64_t ro, j;
    double m;
    double v[RHT ? 16 : 1];
    float vf[RHT ? 1 : 16];
  };
  auto fetch = [&](int64_t it, Item& I) {
    I.live = it < items;
    const int64_t b = it >> 4;   // (16-row group, block) of this half-warp
    // transposed input: consecutive groups are consecutive input columns
    const int64_t g = p.transpose ? b % rg_cov : b / nb_cov;
    I.j = p.transpose ? b / rg_cov : b % nb_cov;
    I.ro = g * 16 + i16;
    I.has = I.live && I.ro < R && I.j < nb;
    I.m = 0.0;
    if (I.has) {
      if constexpr (RHT) {
        load_block(p, I.ro, I.j, I.v);
#pragma unroll
        for (int e = 0; e < 16; ++e) I.m = fmax(I.m, fabs(I.v[e]));
      } else {
        load_block_f32(p, I.ro, I.j, I.vf);
        float mf = 0.0f;
#pragma unroll
        for (int e = 0; e < 16; ++e) mf = fmaxf(mf, fabsf(I.vf[e]));
        I.m = static_cast<double>(mf);
      }
    }
  };
  auto finish = [&](Item& I) {
    double m = I.m;
    if (p.block2d) {   // one scale from the amax of the 16 x 16 block
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
    }
    if (!I.live) return;
    const int64_t ro = I.ro, j = I.j;
    uint32_t scode = 0;
    if (I.has) {
      uint32_t lo = 0, hi = 0;
      float q[16];
      bool nz;
      if constexpr (RHT) {
        scode = cvt_to_e4m3(__double2float_rn(m / static_cast<double>(t)));
        const double dec = e4m3_exact(scode);
        nz = dec != 0.0;
        if (nz) {
          const float sc = __fmul_rn(static_cast<float>(dec), s_g);
#pragma unroll
          for (int e = 0; e < 16; ++e) q[e] = __double2float_rn(I.v[e] / static_cast<double>(sc));
        }
      } else {
        scode = cvt_to_e4m3(__fdiv_rn(static_cast<float>(m), t));
        const float dec = e4m3_exact_f(scode);
        nz = dec != 0.0f;
        if (nz) {
          const float sc = __fmul_rn(dec, s_g);
#pragma unroll
          for (int e = 0; e < 16; ++e) q[e] = __fdiv_rn(I.vf[e], sc);
        }
      }
      if (nz) {
        if (p.sr) {
          float u[16];
          sr_uniforms16(static_cast<uint64_t>(ro) * C + j * 16, p.seed, p.stream, u);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint32_t c = e2m1_sr(q[e], u[e]);
            if (e < 8) lo |= c << (4 * e);
            else hi |= c << (4 * (e - 8));
          }
        } else {   // round to nearest even (hardware conversion, element 2k in the low nibble)
          lo = cvt_e2m1_x8(q);
          hi = cvt_e2m1_x8(q + 8);
        }
      }
      *reinterpret_cast<uint2*>(p.codes + ro * (ld / 2) + j * 8) = make_uint2(lo, hi);
    } else if (ro < R && j < nb_store) {
      *reinterpret_cast<uint2*>(p.codes + ro * (ld / 2) + j * 8) = make_uint2(0u, 0u);
    }
    if (p.tiled) {
      if (ro < ((R + 127) / 128) * 128) p.sf[tiled_off(ro, j, ld64)] = static_cast<uint8_t>(scode);
    } else if (ro < R && j < nb_store) {
      p.sf[ro * (ld / 16) + j] = static_cast<uint8_t>(scode);
    }
  };
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it < items32; it += stride) {
    Item I;
    fetch(it, I);
    finish(I);
  }
}

// Transpose of NVFP4 data with 16 x 16 scale blocks: a CTA per 128 x 128
// tile of one group. The tile's codes (128 rows x 64 bytes) are staged in
// shared memory; thread (c = tid % 128, half = tid / 128) then gathers input
// rows half * 64 .. half * 64 + 63 of column c (64 nibbles, element 2k in the
// low nibble) into 32 bytes of output row c, and writes the four scales of
// those rows' 16-row groups as one word of the output's MMA-tiled layout.
__global__ void __launch_bounds__(256) nvfp4_transpose2d_kernel(const uint8_t* __restrict__ codes,
                                                                 const uint8_t* __restrict__ sf, int64_t rows,
                                                                 int64_t cols, uint8_t* __restrict__ codes_t,
                                                                 uint8_t* __restrict__ sf_t) {
  pdl_begin();
  __shared__ __align__(16) uint8_t tile[128 * 64];
  const int64_t g = blockIdx.z;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 128, c0 = static_cast<int64_t>(blockIdx.x) * 128;
  const uint8_t* in = codes + g * rows * cols / 2;
  const uint8_t* in_sf = sf + g * rows * cols / 16;
  uint8_t* out = codes_t + g * rows * cols / 2;
  uint8_t* out_sf = sf_t + g * rows * cols / 16;
  const int tid = threadIdx.x;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int idx = tid + k * 256;
    const int row = idx >> 2, part = idx & 3;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(in + (r0 + row) * (cols / 2) + c0 / 2) + part);
    *reinterpret_cast<uint4*>(tile + row * 64 + part * 16) = v;
  }
  __syncthreads();
  const int c = tid & 127, half = tid >> 7;
  const int shift = (c & 1) * 4;
  uint32_t w[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t word = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) {   // nibble b of the word: input row half * 64 + q * 8 + b
      const int r = half * 64 + q * 8 + b;
      word |= static_cast<uint32_t>((tile[r * 64 + (c >> 1)] >> shift) & 15u) << (4 * b);
    }
    w[q] = word;
  }
  uint4* dst = reinterpret_cast<uint4*>(out + (c0 + c) * (rows / 2) + r0 / 2 + half * 32);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  // scales: output row c0 + c, blocks j = (r0 + half * 64) / 16 + 0..3
  const int64_t g64_in = cols / 64, g64_out = rows / 64;
  const int64_t jc = (c0 + c) / 16;   // the input's scale column of this output row
  uint32_t sw = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b)
    sw |= static_cast<uint32_t>(__ldg(in_sf + tiled_off(r0 + half * 64 + b * 16, jc, g64_in))) << (8 * b);
  *reinterpret_cast<uint32_t*>(out_sf + tiled_off(c0 + c, (r0 + half * 64) / 16, g64_out)) = sw;
}

}  // namespace

lmoe_status launch_nvfp4_transpose2d(const uint8_t* codes, const uint8_t* sf, int64_t groups, int64_t rows,
                                     int64_t cols, uint8_t* codes_t, uint8_t* sf_t, cudaStream_t s) {
  if (groups < 0 || rows < 0 || cols < 0) return LMOE_ERR_INVALID_ARG;
  if (groups == 0 || rows == 0 || cols == 0) return LMOE_OK;
  if (!codes || !sf || !codes_t || !sf_t) return LMOE_ERR_INVALID_ARG;
  if (rows % 128 || cols % 128 || groups > 65535 || rows / 128 > 65535 || cols / 128 > 0x7fffffff)
    return LMOE_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(codes) | reinterpret_cast<uintptr_t>(codes_t) | reinterpret_cast<uintptr_t>(sf) |
       reinterpret_cast<uintptr_t>(sf_t)) & 15)
    return LMOE_ERR_INVALID_ARG;
  launch_k(nvfp4_transpose2d_kernel, dim3(static_cast<unsigned>(cols / 128), static_cast<unsigned>(rows / 128),
                                          static_cast<unsigned>(groups)),
           dim3(256), 0, s, codes, sf, rows, cols, codes_t, sf_t);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

int nvfp4x_partials(int64_t blocks) {
  const int64_t want = (blocks + 4 * kXThreads - 1) / (4 * kXThreads);
  return static_cast<int>(want < 1 ? 1 : (want > 1184 ? 1184 : want));
}

lmoe_status launch_nvfp4_quantize_ex(const void* in, int in_dtype, int64_t rows, int64_t cols, uint32_t flags,
                                     uint32_t rht_signs, uint64_t seed, uint32_t sr_stream, const float* global_in,
                                     uint8_t* codes, uint8_t* sf, float* global_out, int sf_layout, double* partials,
                                     cudaStream_t s, int64_t out_pitch, int groups) {
  QxParams p = {};
  p.in = in;
  p.bf16 = in_dtype == LMOE_BF16;
  p.rows = rows;
  p.cols = cols;
  p.transpose = (flags & LMOE_QX_TRANSPOSE) != 0;
  p.rht = (flags & LMOE_QX_RHT) != 0;
  p.signs = rht_signs & 0xFFFFu;
  p.sr = (flags & LMOE_QX_SR) != 0;
  p.seed = seed;
  p.stream = sr_stream;
  p.block2d = (sf_layout & LMOE_SF_BLOCK_16X16) != 0;
  p.tiled = (sf_layout & ~LMOE_SF_BLOCK_16X16) == LMOE_SF_MMA_TILED;
  p.global_in = global_in;
  p.codes = codes;
  p.sf = sf;
  p.global_out = global_out;
  p.vec = (reinterpret_cast<uintptr_t>(in) & 15) == 0;
  const int64_t R = p.transpose ? cols : rows, C = p.transpose ? rows : cols;
  p.pitch = out_pitch > 0 ? out_pitch : C;
  if (p.pitch < C || p.pitch % 16) return LMOE_ERR_INVALID_ARG;
  // groups share one SR stream, so stochastic rounding stays one group per launch
  if (groups < 1 || groups > 65535 || (groups > 1 && (p.sr || global_in))) return LMOE_ERR_INVALID_ARG;
  if (R == 0) return LMOE_OK;
  const int64_t groups64 = (p.pitch + 63) / 64;
  p.gs_in = rows * cols;
  p.gs_codes = R * p.pitch / 2;
  p.gs_sf = p.tiled ? (R + 127) / 128 * groups64 * 512 : R * (p.pitch / 16);
  const int sms = device_sm_count();
  const int np = nvfp4x_partials(R * (C / 16));
  if (!global_in) {
    launch_k(p.rht ? qx_amax_kernel<true> : qx_amax_kernel<false>, dim3(np, groups), dim3(kXThreads), 0, s, p, partials);
    count_launch();
  }
  p.partials = partials;
  p.np = global_in ? 0 : np;
  const int64_t rg_cov = p.tiled ? (R + 127) / 128 * 8 : (R + 15) / 16;
  const int64_t nb_cov = p.tiled ? groups64 * 4 : p.pitch / 16;
  int64_t blocks = (rg_cov * nb_cov * 16 + kXThreads - 1) / kXThreads;
  const int64_t cap = (static_cast<int64_t>(sms) * 8 + groups - 1) / groups;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  launch_k(p.rht ? qx_encode_kernel<true> : qx_encode_kernel<false>, dim3(static_cast<unsigned>(blocks), groups),
           dim3(kXThreads), 0, s, p);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

lmoe_status launch_nvfp4_quantize_groups(const void* in, int in_dtype, int64_t rows_max, int64_t cols,
                                         uint32_t flags, uint32_t rht_signs, uint64_t seed, uint32_t stream0,
                                         uint32_t stream_step, const int64_t* gtab, int groups, int64_t pitch_max,
                                         int64_t ld, uint8_t* codes, uint8_t* sf, float* global_out, int sf_layout,
                                         double* partials, cudaStream_t s) {
  if (groups < 1 || groups > 65535 || !gtab || !global_out || rows_max < 0 || cols <= 0 || cols % 16)
    return LMOE_ERR_INVALID_ARG;
  QxParams p = {};
  p.in = in;
  p.bf16 = in_dtype == LMOE_BF16;
  p.rows = rows_max;
  p.cols = cols;
  p.transpose = (flags & LMOE_QX_TRANSPOSE) != 0;
  p.rht = (flags & LMOE_QX_RHT) != 0;
  p.signs = rht_signs & 0xFFFFu;
  p.sr = (flags & LMOE_QX_SR) != 0;
  p.seed = seed;
  p.stream = stream0;
  p.stream_step = stream_step;
  p.block2d = (sf_layout & LMOE_SF_BLOCK_16X16) != 0;
  p.tiled = (sf_layout & ~LMOE_SF_BLOCK_16X16) == LMOE_SF_MMA_TILED;
  p.codes = codes;
  p.sf = sf;
  p.global_out = global_out;
  p.vec = (reinterpret_cast<uintptr_t>(in) & 15) == 0;
  p.gtab = gtab;
  const int64_t R = p.transpose ? cols : rows_max, C = p.transpose ? rows_max : cols;
  const int64_t pitch = pitch_max > C ? pitch_max : C;
  if (pitch % 16 || ld < 0 || ld % 64) return LMOE_ERR_INVALID_ARG;
  p.ld = ld;
  const int sms = device_sm_count();
  const int np = nvfp4x_partials(R * (pitch / 16) > 0 ? R * (pitch / 16) : 1);
  launch_k(p.rht ? qx_amax_kernel<true> : qx_amax_kernel<false>, dim3(np, groups), dim3(kXThreads), 0, s, p, partials);
  count_launch();
  p.partials = partials;
  p.np = np;
  const int64_t rg_cov = p.tiled ? (R + 127) / 128 * 8 : (R + 15) / 16;
  const int64_t nb_cov = p.tiled ? (pitch + 63) / 64 * 4 : pitch / 16;
  int64_t blocks = (rg_cov * nb_cov * 16 + kXThreads - 1) / kXThreads;
  const int64_t cap = (static_cast<int64_t>(sms) * 8 + groups - 1) / groups;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  launch_k(p.rht ? qx_encode_kernel<true> : qx_encode_kernel<false>, dim3(static_cast<unsigned>(blocks), groups),
           dim3(kXThreads), 0, s, p);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

}  // namespace lmoe
