// Backward of the routed experts' FFNs under the NVFP4 training recipe
// (greeksharifa page on the Nemotron 3 whitepaper, section 2.4 "NVFP4
// Training"; notes.yuuk.io page, section 4 "NVFP4 pre-training"): fprop,
// dgrad and wgrad of both expert GEMMs run as block-scaled NVFP4 GEMMs,
// weights quantised with 16 x 16 blocks, gradients rounded stochastically,
// and the two wgrad operands transformed with a random Hadamard transform
// along the tokens (the contraction) before they are quantised.
//
// Per expert e, over its n slot rows (padded with zero rows to R, a multiple
// of 16, wherever a quantiser runs along the tokens):
//   h = zq W1q^T, aq = NVFP4(relu(h)^2, s_a), o = aq W2q^T  (recomputed;
//   h, o and dA kept in fp32: a stochastic quantiser turns any rounding of
//   its input into changed codes, so its inputs stay unrounded)
//   dgate = dy . o per row, do = gate * dy
//   dA = SR(do) W2q,          dW2 = SR(RHT(do)^T) RN(RHT(aq)^T)^T
//   dh = dA * 2 max(h, 0)
//   dz = SR(dh) W1q,          dW1 = SR(RHT(dh)^T) RN(RHT(zq)^T)^T
// with SR uniforms from Philox-4x32-10 on stream 4 e + 2 g + j (g: 0 first
// GEMM, 1 second; j: 0 dgrad, 1 wgrad). The host walks the experts; every
// step is a kernel of this library (the training quantiser, the grouped
// NVFP4 GEMM, and the three small kernels below).
#include <cuda_bf16.h>

#include <vector>

#include "lmoe_device.cuh"
#include "lmoe_internal.h"

namespace lmoe {
namespace {

constexpr int kBwThreads = 256;

size_t up256(size_t b) { return (b + 255) / 256 * 256; }
int64_t ceil_to(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// do[r][:] = gate * dy for r < n (fp32; rows n..R-1 zero); dgate[r] = dy . o.
// A block per row r < R.
__global__ void __launch_bounds__(kBwThreads) bw_prep_kernel(const float* __restrict__ dy,
                                                              const float* __restrict__ o,
                                                              const float* __restrict__ gate, int64_t row0, int n,
                                                              int l, float* __restrict__ d_o,
                                                              float* __restrict__ dgate) {
  pdl_begin();
  __shared__ float red[kBwThreads / 32];
  const int r = blockIdx.x;
  float* out = d_o + static_cast<int64_t>(r) * l;
  if (r >= n) {
    for (int j = threadIdx.x; j < l; j += blockDim.x) out[j] = 0.0f;
    return;
  }
  const int64_t row = row0 + r;
  const float g = __ldg(gate + row);
  float dot = 0.0f;
  for (int j = threadIdx.x; j < l; j += blockDim.x) {
    const float d = dy[row * l + j];
    dot = fmaf(d, o[row * l + j], dot);
    out[j] = __fmul_rn(g, d);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = dot;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.0f;
    for (int i = 0; i < kBwThreads / 32; ++i) s += red[i];
    dgate[row] = s;
  }
}

// dh[r][c] = dA[r][c] * 2 max(h[row0 + r][c], 0) for r < n, 0 for n <= r < R.
__global__ void __launch_bounds__(kBwThreads) bw_dh_kernel(const float* __restrict__ dA,
                                                            const float* __restrict__ h, int64_t row0,
                                                            int n, int R, int m, float* __restrict__ dh) {
  pdl_begin();
  const int64_t total = static_cast<int64_t>(R) * m;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / m, c = i % m;
    float v = 0.0f;
    if (r < n) {
      v = dA[r * m + c] * (2.0f * fmaxf(h[(row0 + r) * m + c], 0.0f));
    }
    dh[i] = v;
  }
}

// E2M1 magnitude by code (0, 0.5, 1, 1.5, 2, 3, 4, 6).
__device__ __forceinline__ double e2m1_mag(uint32_t c) {
  return (c < 4) ? 0.5 * static_cast<double>(c) : (c < 6 ? static_cast<double>(c - 2) : (c == 6 ? 4.0 : 6.0));
}

// E4M3 code -> value: subnormal f * 2^-9, normal (8 + f) * 2^(e - 10).
__device__ __forceinline__ double e4m3_val(uint32_t c) {
  const int e = (c >> 3) & 15, f = c & 7;
  return e == 0 ? ldexp(static_cast<double>(f), -9) : ldexp(static_cast<double>(8 + f), e - 10);
}

// Rows row0 .. row0 + R - 1 of NVFP4 codes [*, cols/2] with MMA-tiled scales
// (groups64 = cols / 64) and a global scale, as fp32 [R][cols]; rows >= n are
// zero. Each value is code * block scale * global, formed exactly in fp64
// (2 + 4 + 24 significant bits) and rounded once to fp32.
__global__ void __launch_bounds__(kBwThreads) bw_dequant_kernel(const uint8_t* __restrict__ codes,
                                                                 const uint8_t* __restrict__ sf,
                                                                 const float* __restrict__ global, int64_t row0,
                                                                 int n, int R, int cols, float* __restrict__ out) {
  pdl_begin();
  const double s_g = static_cast<double>(__ldg(global));
  const int groups64 = cols / 64;
  const int64_t total = static_cast<int64_t>(R) * (cols / 2);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / (cols / 2);
    const int cb = static_cast<int>(i % (cols / 2));   // byte: elements 2 cb, 2 cb + 1
    float v0 = 0.0f, v1 = 0.0f;
    if (r < n) {
      const int64_t row = row0 + r;
      const uint32_t b = codes[row * (cols / 2) + cb];
      const int j = (2 * cb) / 16;
      const int64_t so = ((row >> 7) * groups64 + (j >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (j & 3);
      const double sc = e4m3_val(sf[so]) * s_g;
      const uint32_t c0 = b & 15u, c1 = b >> 4;
      v0 = __double2float_rn((c0 & 8u ? -1.0 : 1.0) * e2m1_mag(c0 & 7u) * sc);
      v1 = __double2float_rn((c1 & 8u ? -1.0 : 1.0) * e2m1_mag(c1 & 7u) * sc);
    }
    out[r * cols + 2 * cb] = v0;
    out[r * cols + 2 * cb + 1] = v1;
  }
}

unsigned grid_for(int64_t items) {
  const int64_t sms = device_sm_count();
  int64_t b = (items + kBwThreads - 1) / kBwThreads;
  if (b > sms * 8) b = sms * 8;
  return static_cast<unsigned>(b < 1 ? 1 : b);
}

// Workspace carve-up (all offsets 256-byte aligned).
struct BwLayout {
  size_t err, w1c, w1s, w1g, w2c, w2s, w2g, w1tc, w1ts, w1tg, w2tc, w2ts, w2tg, h, aqc, aqs, o, d_o, dh, deq, qac, qas, qag, dA,
      t1c, t1s, t1g, t2c, t2s, t2g, part, tab, total;
  int64_t P, Rmax, R128max, K256max;
};

// P: padded slot rows; Rmax: the largest expert's rows rounded up to 16.
BwLayout bw_layout_for(const lmoe_config* c, int64_t P, int64_t Rmax) {
  BwLayout L = {};
  const int64_t N = c->N, l = c->l, m = c->m;
  L.P = P;
  L.Rmax = Rmax;
  L.R128max = ceil_to(Rmax, 128);
  L.K256max = ceil_to(Rmax, 256);
  const int64_t lm = l > m ? l : m;
  size_t off = 0;
  auto take = [&](size_t b) {
    const size_t o = off;
    off += up256(b);
    return o;
  };
  L.err = take(256);
  L.w1c = take(N * m * l / 2);
  L.w1s = take(N * m * l / 16);
  L.w1g = take(N * 4);
  L.w2c = take(N * l * m / 2);
  L.w2s = take(N * l * m / 16);
  L.w2g = take(N * 4);
  L.w1tc = take(N * l * m / 2);   // transposed weights (dgrad operands), every expert
  L.w1ts = take(N * l * m / 16);
  L.w1tg = take(N * 4);
  L.w2tc = take(N * l * m / 2);
  L.w2ts = take(N * l * m / 16);
  L.w2tg = take(N * 4);
  L.h = take(P * m * 4);
  L.aqc = take(P * m / 2);
  L.aqs = take(P * m / 16);
  L.o = take(P * l * 4);
  L.d_o = take(Rmax * l * 4);
  L.dh = take(Rmax * m * 4);
  L.deq = take(Rmax * lm * 4);
  L.qac = take(L.R128max * lm / 2);
  L.qas = take(L.R128max * lm / 16);
  L.qag = take(4);
  L.dA = take(L.R128max * m * 4);
  L.t1c = take(lm * L.K256max / 2);
  L.t1s = take(lm * L.K256max / 16);
  L.t1g = take(4);
  L.t2c = take(lm * L.K256max / 2);
  L.t2s = take(lm * L.K256max / 16);
  L.t2g = take(4);
  // amax partials: the grouped weight launches (N groups) or one gradient operand
  const int64_t np_w = N * nvfp4x_partials(m * l / 16 > 0 ? m * l / 16 : 1);
  const int64_t np_g = nvfp4x_partials(Rmax * lm / 16 > 0 ? Rmax * lm / 16 : 1);
  L.part = take(static_cast<size_t>(np_w > np_g ? np_w : np_g) * 8);
  L.tab = take((N * 4 + 8) * 4);   // per expert {0, n, 0, R128}; then {0, l, 0, l}, {0, m, 0, m}
  L.total = off;
  return L;
}

BwLayout bw_layout(const lmoe_config* c, const int32_t* counts) {
  int64_t P = 0, Rmax = 0;
  for (int e = 0; e < c->N; ++e) {
    P += ceil_to(counts[e], 128);
    if (counts[e] > 0 && ceil_to(counts[e], 16) > Rmax) Rmax = ceil_to(counts[e], 16);
  }
  return bw_layout_for(c, P, Rmax);
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace lmoe

using namespace lmoe;

extern "C" {

size_t lmoe_expert_backward_nvfp4_workspace(const lmoe_config* cfg, const int32_t* counts) {
  if (!cfg || !counts || cfg->N <= 0 || cfg->l <= 0 || cfg->m <= 0) return 0;
  for (int e = 0; e < cfg->N; ++e)
    if (counts[e] < 0) return 0;
  return bw_layout(cfg, counts).total;
}

lmoe_status lmoe_expert_backward_nvfp4(const lmoe_config* cfg, const int32_t* counts, const int32_t* offsets,
                                       const int32_t* padded_offsets, const uint8_t* z_codes, const uint8_t* z_sf,
                                       const float* z_global, const void* w1, const void* w2,
                                       const float* a_global, const float* gate, const float* dy, uint64_t seed,
                                       uint32_t rht_signs, void* dz, float* dgate, void* dw1, void* dw2, void* ws,
                                       size_t ws_bytes, void* stream) {
  if (!cfg || !counts || !offsets || !padded_offsets || !z_codes || !z_sf || !z_global || !w1 || !w2 ||
      !a_global || !gate || !dy || !dz || !dgate || !dw1 || !dw2)
    return LMOE_ERR_INVALID_ARG;
  const int N = cfg->N;
  const int64_t l = cfg->l, m = cfg->m;
  if (N <= 0 || N > 1024 || l <= 0 || m <= 0) return LMOE_ERR_INVALID_ARG;
  if (l % 256 || m % 256) return LMOE_ERR_UNSUPPORTED;
  for (int e = 0; e < N; ++e)
    if (counts[e] < 0) return LMOE_ERR_INVALID_ARG;
  if (!a16(z_codes) || !a16(z_sf) || !a16(w1) || !a16(w2) || !a16(dy) || !a16(dz) || !a16(dw1) || !a16(dw2))
    return LMOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < bw_layout(cfg, counts).total) return LMOE_ERR_WORKSPACE;
  return expert_backward_core(cfg, counts, offsets, padded_offsets, z_codes, z_sf, z_global, w1, w2, a_global, gate,
                              dy, seed, rht_signs, dz, dgate, dw1, dw2, ws, nullptr, nullptr,
                              static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace lmoe {

size_t expert_backward_ws(const lmoe_config* cfg, const int32_t* counts) { return bw_layout(cfg, counts).total; }

// Enough for any routing of cfg->T tokens: at most padded_rows slot rows, and
// no expert with more than T rows (a token picks an expert once).
size_t expert_backward_ws_bound(const lmoe_config* cfg) {
  return bw_layout_for(cfg, lmoe_padded_rows(cfg), ceil_to(cfg->T > 0 ? cfg->T : 1, 16)).total;
}

// The routed experts' backward (see lmoe_expert_backward_nvfp4), arguments
// checked by the caller; ws holds at least expert_backward_ws() bytes. With
// o_out, the recomputed expert outputs o (fp32, [P][l]) are copied there.
lmoe_status expert_backward_core(const lmoe_config* cfg, const int32_t* counts, const int32_t* offsets,
                                 const int32_t* padded_offsets, const uint8_t* z_codes, const uint8_t* z_sf,
                                 const float* z_global, const void* w1, const void* w2, const float* a_global,
                                 const float* gate, const float* dy, uint64_t seed, uint32_t rht_signs, void* dz,
                                 float* dgate, void* dw1, void* dw2, void* ws, float* o_out, uint32_t* err_word,
                                 cudaStream_t s) {
  const int N = cfg->N;
  const int64_t l = cfg->l, m = cfg->m;
  const BwLayout L = bw_layout(cfg, counts);
  uint32_t* err = err_word ? err_word : at<uint32_t>(ws, L.err);
  double* part = at<double>(ws, L.part);
  lmoe_status st = LMOE_OK;
  const __nv_bfloat16* W1 = static_cast<const __nv_bfloat16*>(w1);
  const __nv_bfloat16* W2 = static_cast<const __nv_bfloat16*>(w2);
  const int tiled2d = LMOE_SF_MMA_TILED | LMOE_SF_BLOCK_16X16;

  // per-expert GEMM offsets: {0, n, 0, R128}; wgrad problems {0, l, 0, l} and {0, m, 0, m}
  std::vector<int32_t> tab(static_cast<size_t>(N) * 4 + 8);
  std::vector<int64_t> poff(N + 1, 0);
  for (int e = 0; e < N; ++e) {
    const int64_t n = counts[e];
    tab[4 * e + 0] = 0;
    tab[4 * e + 1] = static_cast<int32_t>(n);
    tab[4 * e + 2] = 0;
    tab[4 * e + 3] = static_cast<int32_t>(ceil_to(ceil_to(n, 16), 128));
    poff[e + 1] = poff[e] + ceil_to(n, 128);
  }
  int32_t* tail = tab.data() + 4 * N;
  tail[0] = 0;
  tail[1] = static_cast<int32_t>(l);
  tail[2] = 0;
  tail[3] = static_cast<int32_t>(l);
  tail[4] = 0;
  tail[5] = static_cast<int32_t>(m);
  tail[6] = 0;
  tail[7] = static_cast<int32_t>(m);
  int32_t* dtab = at<int32_t>(ws, L.tab);
  if (cudaMemcpyAsync(dtab, tab.data(), tab.size() * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return LMOE_ERR_CUDA;
  const int32_t* off_l = dtab + 4 * N;       // {0, l}
  const int32_t* off_m = dtab + 4 * N + 4;   // {0, m}

  // every expert's weights with 16 x 16 blocks (current amax per expert and
  // matrix), one grouped launch each: W1 [m][l] and W2 [l][m] for the forward,
  // W2^T [m][l] and W1^T [l][m] for the dgrads
  if ((st = launch_nvfp4_quantize_ex(W1, LMOE_BF16, m, l, 0, 0, 0, 0, nullptr, at<uint8_t>(ws, L.w1c),
                                     at<uint8_t>(ws, L.w1s), at<float>(ws, L.w1g), tiled2d, part, s, 0, N)) !=
      LMOE_OK)
    return st;
  if ((st = launch_nvfp4_quantize_ex(W2, LMOE_BF16, l, m, 0, 0, 0, 0, nullptr, at<uint8_t>(ws, L.w2c),
                                     at<uint8_t>(ws, L.w2s), at<float>(ws, L.w2g), tiled2d, part, s, 0, N)) !=
      LMOE_OK)
    return st;
  if ((st = launch_nvfp4_quantize_ex(W2, LMOE_BF16, l, m, LMOE_QX_TRANSPOSE, 0, 0, 0, nullptr,
                                     at<uint8_t>(ws, L.w2tc), at<uint8_t>(ws, L.w2ts), at<float>(ws, L.w2tg), tiled2d,
                                     part, s, 0, N)) != LMOE_OK)
    return st;
  if ((st = launch_nvfp4_quantize_ex(W1, LMOE_BF16, m, l, LMOE_QX_TRANSPOSE, 0, 0, 0, nullptr,
                                     at<uint8_t>(ws, L.w1tc), at<uint8_t>(ws, L.w1ts), at<float>(ws, L.w1tg), tiled2d,
                                     part, s, 0, N)) != LMOE_OK)
    return st;

  // recomputed forward over all slots: h (BF16), aq (NVFP4 with the static s_a), o (BF16)
  Fp4Launch f;
  f.a_codes = z_codes;
  f.a_sf = z_sf;
  f.a_rows = L.P;
  f.b_codes = at<uint8_t>(ws, L.w1c);
  f.b_sf = at<uint8_t>(ws, L.w1s);
  f.k = l;
  f.cols = static_cast<int>(m);
  f.groups = N;
  f.offsets = offsets;
  f.padded_offsets = padded_offsets;
  f.in_scale = z_global;
  f.w_scale = at<float>(ws, L.w1g);
  f.out = at<void>(ws, L.h);
  f.ld_out = m;
  f.f32_out = 1;
  if (L.P > 0 && (st = fp4_gemm(f, err, s)) != LMOE_OK) return st;
  Fp4Launch fq = f;
  fq.quant_out = 1;
  fq.f32_out = 0;
  fq.out_scale = a_global;
  fq.out = at<void>(ws, L.aqc);
  fq.out_sf = at<uint8_t>(ws, L.aqs);
  if (L.P > 0 && (st = fp4_gemm(fq, err, s)) != LMOE_OK) return st;
  Fp4Launch f2 = f;   // fp32 out, as f
  f2.a_codes = at<uint8_t>(ws, L.aqc);
  f2.a_sf = at<uint8_t>(ws, L.aqs);
  f2.b_codes = at<uint8_t>(ws, L.w2c);
  f2.b_sf = at<uint8_t>(ws, L.w2s);
  f2.k = m;
  f2.cols = static_cast<int>(l);
  f2.in_scale = a_global;
  f2.w_scale = at<float>(ws, L.w2g);
  f2.out = at<void>(ws, L.o);
  f2.ld_out = l;
  if (L.P > 0 && (st = fp4_gemm(f2, err, s)) != LMOE_OK) return st;

  float* d_o = at<float>(ws, L.d_o);
  float* dh = at<float>(ws, L.dh);
  float* deq = at<float>(ws, L.deq);
  uint8_t *qac = at<uint8_t>(ws, L.qac), *qas = at<uint8_t>(ws, L.qas);
  float* qag = at<float>(ws, L.qag);
  uint8_t *t1c = at<uint8_t>(ws, L.t1c), *t1s = at<uint8_t>(ws, L.t1s);
  uint8_t *t2c = at<uint8_t>(ws, L.t2c), *t2s = at<uint8_t>(ws, L.t2s);
  float *t1g = at<float>(ws, L.t1g), *t2g = at<float>(ws, L.t2g);
  float* dA = at<float>(ws, L.dA);
  const float* h = at<float>(ws, L.h);
  const float* o = at<float>(ws, L.o);

  // a single-group GEMM out[rows][cols] = A[rows][k] . B[cols][k]^T (BF16 out)
  auto gemm1 = [&](const uint8_t* ac, const uint8_t* as, const float* ag, int64_t a_rows, const int32_t* off,
                   const uint8_t* bc, const uint8_t* bs, const float* bg, int64_t cols, int64_t k, void* out,
                   int64_t ld, int f32) {
    Fp4Launch g;
    g.a_codes = ac;
    g.a_sf = as;
    g.a_rows = a_rows;
    g.b_codes = bc;
    g.b_sf = bs;
    g.k = k;
    g.cols = static_cast<int>(cols);
    g.groups = 1;
    g.offsets = off;
    g.padded_offsets = off + 2;
    g.in_scale = ag;
    g.w_scale = bg;
    g.out = out;
    g.ld_out = ld;
    g.f32_out = f32;
    return fp4_gemm(g, err, s);
  };

  for (int e = 0; e < N && st == LMOE_OK; ++e) {
    const int n = counts[e];
    if (n == 0) {   // no rows: zero weight gradients
      if (cudaMemsetAsync(static_cast<__nv_bfloat16*>(dw1) + e * m * l, 0, m * l * 2, s) != cudaSuccess ||
          cudaMemsetAsync(static_cast<__nv_bfloat16*>(dw2) + e * l * m, 0, l * m * 2, s) != cudaSuccess)
        return LMOE_ERR_CUDA;
      continue;
    }
    const int R = static_cast<int>(ceil_to(n, 16));
    const int64_t R128 = ceil_to(R, 128), K256 = ceil_to(R, 256);
    const int64_t p0 = poff[e];
    const int32_t* off_e = dtab + 4 * e;
    const uint32_t st_dg1 = 4u * e + 0, st_wg1 = 4u * e + 1, st_dg2 = 4u * e + 2, st_wg2 = 4u * e + 3;

    // do, dgate
    launch_k(bw_prep_kernel, dim3(R), dim3(kBwThreads), 0, s, static_cast<const float*>(dy), o, gate, p0, n,
             static_cast<int>(l), d_o, dgate);
    count_launch();
    // second GEMM, dgrad: dA = SR(do) W2q  (W2^T [m][l] with 16 x 16 blocks)
    if ((st = launch_nvfp4_quantize_ex(d_o, LMOE_F32, R, l, LMOE_QX_SR, rht_signs, seed, st_dg2, nullptr, qac, qas,
                                       qag, LMOE_SF_MMA_TILED, part, s)) != LMOE_OK)
      break;
    if ((st = gemm1(qac, qas, qag, R128, off_e, at<uint8_t>(ws, L.w2tc) + e * l * m / 2,
                    at<uint8_t>(ws, L.w2ts) + e * l * m / 16, at<float>(ws, L.w2tg) + e, m, l, dA, m, 1)) != LMOE_OK)
      break;
    // dh
    launch_k(bw_dh_kernel, dim3(grid_for(static_cast<int64_t>(R) * m)), dim3(kBwThreads), 0, s, dA, h, p0, n, R,
             static_cast<int>(m), dh);
    count_launch();
    // second GEMM, wgrad: dW2 = SR(RHT(do)^T) RN(RHT(aq)^T)^T  (contraction over R tokens, stored K256 wide)
    launch_k(bw_dequant_kernel, dim3(grid_for(static_cast<int64_t>(R) * m / 2)), dim3(kBwThreads), 0, s,
             static_cast<const uint8_t*>(at<uint8_t>(ws, L.aqc)), static_cast<const uint8_t*>(at<uint8_t>(ws, L.aqs)),
             a_global, p0, n, R, static_cast<int>(m), deq);
    count_launch();
    if ((st = launch_nvfp4_quantize_ex(d_o, LMOE_F32, R, l, LMOE_QX_TRANSPOSE | LMOE_QX_RHT | LMOE_QX_SR, rht_signs,
                                       seed, st_wg2, nullptr, t1c, t1s, t1g, LMOE_SF_MMA_TILED, part, s, K256)) !=
        LMOE_OK)
      break;
    if ((st = launch_nvfp4_quantize_ex(deq, LMOE_F32, R, m, LMOE_QX_TRANSPOSE | LMOE_QX_RHT, rht_signs, seed, 0,
                                       nullptr, t2c, t2s, t2g, LMOE_SF_MMA_TILED, part, s, K256)) != LMOE_OK)
      break;
    if ((st = gemm1(t1c, t1s, t1g, l, off_l, t2c, t2s, t2g, m, K256, static_cast<__nv_bfloat16*>(dw2) + e * l * m,
                    m, 0)) != LMOE_OK)
      break;
    // first GEMM, dgrad: dz = SR(dh) W1q  (W1^T [l][m] with 16 x 16 blocks), into the expert's slot rows
    if ((st = launch_nvfp4_quantize_ex(dh, LMOE_F32, R, m, LMOE_QX_SR, rht_signs, seed, st_dg1, nullptr, qac, qas,
                                       qag, LMOE_SF_MMA_TILED, part, s)) != LMOE_OK)
      break;
    if ((st = gemm1(qac, qas, qag, R128, off_e, at<uint8_t>(ws, L.w1tc) + e * l * m / 2,
                    at<uint8_t>(ws, L.w1ts) + e * l * m / 16, at<float>(ws, L.w1tg) + e, l, m,
                    static_cast<__nv_bfloat16*>(dz) + p0 * l, l, 0)) != LMOE_OK)
      break;
    // first GEMM, wgrad: dW1 = SR(RHT(dh)^T) RN(RHT(zq)^T)^T
    launch_k(bw_dequant_kernel, dim3(grid_for(static_cast<int64_t>(R) * l / 2)), dim3(kBwThreads), 0, s, z_codes,
             z_sf, z_global, p0, n, R, static_cast<int>(l), deq);
    count_launch();
    if ((st = launch_nvfp4_quantize_ex(dh, LMOE_F32, R, m, LMOE_QX_TRANSPOSE | LMOE_QX_RHT | LMOE_QX_SR, rht_signs,
                                       seed, st_wg1, nullptr, t1c, t1s, t1g, LMOE_SF_MMA_TILED, part, s, K256)) !=
        LMOE_OK)
      break;
    if ((st = launch_nvfp4_quantize_ex(deq, LMOE_F32, R, l, LMOE_QX_TRANSPOSE | LMOE_QX_RHT, rht_signs, seed, 0,
                                       nullptr, t2c, t2s, t2g, LMOE_SF_MMA_TILED, part, s, K256)) != LMOE_OK)
      break;
    st = gemm1(t1c, t1s, t1g, m, off_m, t2c, t2s, t2g, l, K256, static_cast<__nv_bfloat16*>(dw1) + e * m * l, l, 0);
  }
  if (st != LMOE_OK) return st;
  if (o_out && L.P > 0 &&
      cudaMemcpyAsync(o_out, o, static_cast<size_t>(L.P) * l * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return LMOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

}  // namespace lmoe
