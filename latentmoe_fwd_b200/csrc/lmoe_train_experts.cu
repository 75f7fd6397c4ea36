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
// GEMM, 1 second; j: 0 dgrad, 1 wgrad). Every step runs as one launch over
// all experts: the quantiser with a group per expert (its own global scale
// and SR stream), the grouped NVFP4 GEMM for the forward recompute and both
// dgrads, its K-batched form for the wgrads (each expert contracts over its
// own token count), and the three small kernels below with a grid row per
// expert.
#include <cuda_bf16.h>

#include <vector>

#include "lmoe_device.cuh"
#include "lmoe_internal.h"

namespace lmoe {
namespace {

constexpr int kBwThreads = 256;

size_t up256(size_t b) { return (b + 255) / 256 * 256; }
int64_t ceil_to(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// Per expert e (blockIdx.y), etab[4e..4e+3] = {first padded row p0, rows n,
// rows R (n rounded up to 16), first wgrad K column}.

// do[p0 + r][:] = gate * dy for r < n (fp32; rows n..R-1 zero); dgate[p0 + r]
// = dy . o. A block per row. dy is the slot row's upstream gradient: row
// p0 + r of `dy`, or with dy_tok the row of the slot's token (the slot at
// sorted position offsets[e] + r, token perm_src[...] / K) of the token-major
// dy_tok.
__global__ void __launch_bounds__(kBwThreads) bw_prep_kernel(const float* __restrict__ dy,
                                                              const float* __restrict__ o,
                                                              const float* __restrict__ gate,
                                                              const int64_t* __restrict__ etab, int l,
                                                              float* __restrict__ d_o, float* __restrict__ dgate,
                                                              const float* __restrict__ dy_tok,
                                                              const int32_t* __restrict__ perm_src,
                                                              const int32_t* __restrict__ offsets, int K) {
  pdl_begin();
  __shared__ float red[kBwThreads / 32];
  const int64_t* t = etab + 4 * blockIdx.y;
  const int64_t p0 = t[0], n = t[1], R = t[2];
  for (int64_t r = blockIdx.x; r < R; r += gridDim.x) {
    const int64_t row = p0 + r;
    float* out = d_o + row * l;
    if (r >= n) {
      for (int j = threadIdx.x; j < l / 4; j += blockDim.x) reinterpret_cast<float4*>(out)[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    const float g = __ldg(gate + row);
    float dot = 0.0f;
    // 16-byte accesses (l is a multiple of 256)
    const float* dyr = dy_tok ? dy_tok + static_cast<int64_t>(__ldg(perm_src + __ldg(offsets + blockIdx.y) + r) / K) * l
                              : dy + row * l;
    const float4* dy4 = reinterpret_cast<const float4*>(dyr);
    const float4* o4 = reinterpret_cast<const float4*>(o + row * l);
    float4* out4 = reinterpret_cast<float4*>(out);
    for (int j = threadIdx.x; j < l / 4; j += blockDim.x) {
      const float4 d = dy4[j], v = o4[j];
      dot = fmaf(d.x, v.x, dot);
      dot = fmaf(d.y, v.y, dot);
      dot = fmaf(d.z, v.z, dot);
      dot = fmaf(d.w, v.w, dot);
      out4[j] = make_float4(__fmul_rn(g, d.x), __fmul_rn(g, d.y), __fmul_rn(g, d.z), __fmul_rn(g, d.w));
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
    __syncthreads();   // red is reused by the block's next row
  }
}

// dh[p0 + r][c] = dA[p0 + r][c] * 2 max(h[p0 + r][c], 0) for r < n, 0 for n <= r < R.
__global__ void __launch_bounds__(kBwThreads) bw_dh_kernel(const float* __restrict__ dA,
                                                            const float* __restrict__ h,
                                                            const int64_t* __restrict__ etab, int m,
                                                            float* __restrict__ dh) {
  pdl_begin();
  const int64_t* t = etab + 4 * blockIdx.y;
  const int64_t p0 = t[0], n = t[1], R = t[2];
  const int64_t total = R * m / 4;   // float4 groups (m is a multiple of 256)
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = (4 * i) / m;
    const int64_t at = p0 * m / 4 + i;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < n) {
      const float4 a = reinterpret_cast<const float4*>(dA)[at], hv = reinterpret_cast<const float4*>(h)[at];
      v = make_float4(a.x * (2.0f * fmaxf(hv.x, 0.0f)), a.y * (2.0f * fmaxf(hv.y, 0.0f)),
                      a.z * (2.0f * fmaxf(hv.z, 0.0f)), a.w * (2.0f * fmaxf(hv.w, 0.0f)));
    }
    reinterpret_cast<float4*>(dh)[at] = v;
  }
}

// Rows p0 .. p0 + R - 1 of NVFP4 codes [*, cols/2] with MMA-tiled scales
// (groups64 = cols / 64) and a global scale, as fp32 [*][cols] at the same
// rows; rows >= p0 + n are zero. A thread per 16-element block. Each value is
// code * block scale * global rounded once to fp32: code * block scale has at
// most 6 significant bits, so it is exact in fp32 and one fp32 multiplication
// by the global scale rounds the exact product.
__global__ void __launch_bounds__(kBwThreads) bw_dequant_kernel(const uint8_t* __restrict__ codes,
                                                                 const uint8_t* __restrict__ sf,
                                                                 const float* __restrict__ global,
                                                                 const int64_t* __restrict__ etab, int cols,
                                                                 float* __restrict__ out) {
  pdl_begin();
  const int64_t* t = etab + 4 * blockIdx.y;
  const int64_t p0 = t[0], n = t[1], R = t[2];
  const float s_g = __ldg(global);
  const int nb = cols / 16, groups64 = cols / 64;
  const int64_t total = R * nb;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / nb;
    const int j = static_cast<int>(i % nb);
    const int64_t row = p0 + r;
    float4* dst = reinterpret_cast<float4*>(out + row * cols + j * 16);
    if (r >= n) {
#pragma unroll
      for (int q = 0; q < 4; ++q) dst[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    const uint2 b = __ldg(reinterpret_cast<const uint2*>(codes + row * (cols / 2) + j * 8));
    const int64_t so = ((row >> 7) * groups64 + (j >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (j & 3);
    const uint32_t sc = __ldg(sf + so);
    const int e = (sc >> 3) & 15, f = sc & 7;
    const float dec = static_cast<float>(e == 0 ? f : 8 + f) * __int_as_float(((e == 0 ? -9 : e - 10) + 127) << 23);
    float v[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t c = ((k < 8 ? b.x : b.y) >> (4 * (k & 7))) & 15u;
      const uint32_t m = c & 7u;   // E2M1 magnitude 0, 0.5, 1, 1.5, 2, 3, 4, 6
      const float mag = m < 4 ? 0.5f * static_cast<float>(m) : (m < 6 ? static_cast<float>(m - 2) : (m == 6 ? 4.0f : 6.0f));
      v[k] = __fmul_rn((c & 8u) ? -(mag * dec) : mag * dec, s_g);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  }
}

// Grid for a per-expert loop over `items` (x), one row per expert (y): about
// eight resident CTAs per SM over all experts.
dim3 grid_per_expert(int64_t items, int N) {
  const int64_t sms = device_sm_count();
  int64_t b = (items + kBwThreads - 1) / kBwThreads;
  const int64_t cap = (sms * 8 + N - 1) / N;
  if (b > cap) b = cap;
  return dim3(static_cast<unsigned>(b < 1 ? 1 : b), static_cast<unsigned>(N));
}

// Workspace carve-up (all offsets 256-byte aligned).
struct BwLayout {
  size_t err, w1c, w1s, w1g, w2c, w2s, w2g, w1tc, w1ts, w2tc, w2ts, h, aqc, aqs, o, d_o, dh, deq, qac,
      qas, qag, dA, t1c, t1s, t1g, t2c, t2s, t2g, part, etab, gtab, ktab, total;
  int64_t P, Rmax, Ksum;
};

// P: padded slot rows; Rmax: the largest expert's rows rounded up to 16;
// Ksum: the experts' wgrad contraction lengths (rows rounded up to 256), summed.
BwLayout bw_layout_for(const lmoe_config* c, int64_t P, int64_t Rmax, int64_t Ksum) {
  BwLayout L = {};
  const int64_t N = c->N, l = c->l, m = c->m;
  L.P = P;
  L.Rmax = Rmax;
  L.Ksum = Ksum;
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
  L.w2tc = take(N * l * m / 2);
  L.w2ts = take(N * l * m / 16);
  // every expert's rows at its padded offset
  L.h = take(P * m * 4);
  L.aqc = take(P * m / 2);
  L.aqs = take(P * m / 16);
  L.o = take(P * l * 4);
  L.d_o = take(P * l * 4);
  L.dh = take(P * m * 4);
  L.deq = take(P * lm * 4);   // dequantised wgrad inputs aq, zq
  L.qac = take(P * lm / 2);
  L.qas = take(P * lm / 16);
  L.qag = take(N * 4);
  L.dA = take(P * m * 4);
  // wgrad operands: [lm][Ksum] matrices, expert e's K256_e columns at its offset
  L.t1c = take(lm * Ksum / 2);
  L.t1s = take(lm * Ksum / 16);
  L.t1g = take(N * 4);
  L.t2c = take(lm * Ksum / 2);
  L.t2s = take(lm * Ksum / 16);
  L.t2g = take(N * 4);
  // amax partials of the largest grouped quantiser launch
  const int64_t K256max = ceil_to(Rmax, 256);
  int64_t np = N * nvfp4x_partials(m * l / 16 > 0 ? m * l / 16 : 1);
  const int64_t np_rows = N * nvfp4x_partials(Rmax * lm / 16 > 0 ? Rmax * lm / 16 : 1);
  const int64_t np_t = N * nvfp4x_partials(lm * K256max / 16 > 0 ? lm * K256max / 16 : 1);
  if (np_rows > np) np = np_rows;
  if (np_t > np) np = np_t;
  L.part = take(static_cast<size_t>(np) * 8);
  L.etab = take(N * 4 * 8);       // per expert {p0, n, R, K offset}
  L.gtab = take(6 * N * 6 * 8);   // six quantiser group tables
  L.ktab = take(N * 2 * 4);       // wgrad K range per expert
  L.total = off;
  return L;
}

BwLayout bw_layout(const lmoe_config* c, const int32_t* counts) {
  int64_t P = 0, Rmax = 0, Ksum = 0;
  for (int e = 0; e < c->N; ++e) {
    P += ceil_to(counts[e], 128);
    Ksum += ceil_to(counts[e], 256);
    if (counts[e] > 0 && ceil_to(counts[e], 16) > Rmax) Rmax = ceil_to(counts[e], 16);
  }
  return bw_layout_for(c, P, Rmax, Ksum);
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
  const int64_t P = lmoe_padded_rows(cfg);
  // ceil256(n) <= ceil128(n) + 128 for every expert
  return bw_layout_for(cfg, P, ceil_to(cfg->T > 0 ? cfg->T : 1, 16), P + 128 * static_cast<int64_t>(cfg->N)).total;
}

// The routed experts' backward (see lmoe_expert_backward_nvfp4), arguments
// checked by the caller; ws holds at least expert_backward_ws() bytes. With
// o_out, the recomputed expert outputs o (fp32, [P][l]) are copied there.
lmoe_status expert_backward_core(const lmoe_config* cfg, const int32_t* counts, const int32_t* offsets,
                                 const int32_t* padded_offsets, const uint8_t* z_codes, const uint8_t* z_sf,
                                 const float* z_global, const void* w1, const void* w2, const float* a_global,
                                 const float* gate, const float* dy, uint64_t seed, uint32_t rht_signs, void* dz,
                                 float* dgate, void* dw1, void* dw2, void* ws, float* o_out, uint32_t* err_word,
                                 cudaStream_t s, const float* dy_tok, const int32_t* perm_src, int K) {
  const int N = cfg->N;
  const int64_t l = cfg->l, m = cfg->m;
  const BwLayout L = bw_layout(cfg, counts);
  uint32_t* err = err_word ? err_word : at<uint32_t>(ws, L.err);
  double* part = at<double>(ws, L.part);
  lmoe_status st = LMOE_OK;
  const __nv_bfloat16* W1 = static_cast<const __nv_bfloat16*>(w1);
  const __nv_bfloat16* W2 = static_cast<const __nv_bfloat16*>(w2);
  const int tiled2d = LMOE_SF_MMA_TILED | LMOE_SF_BLOCK_16X16;

  // per expert {p0, n, R, K offset}; six quantiser group tables {first input
  // row, rows, codes offset, scales offset, pitch}: 0 SR(do), 1 RHT(do)^T,
  // 2 RHT(aq)^T, 3 SR(dh), 4 RHT(dh)^T, 5 RHT(zq)^T
  std::vector<int64_t> etab(static_cast<size_t>(N) * 4), gtab(static_cast<size_t>(6) * N * 6);
  std::vector<int32_t> ktab(static_cast<size_t>(N) * 2);   // wgrad K range per expert: {first column, blocks}
  int64_t p0 = 0, koff = 0;
  for (int e = 0; e < N; ++e) {
    const int64_t n = counts[e], R = ceil_to(n, 16), K256 = ceil_to(n, 256);
    etab[4 * e + 0] = p0;
    etab[4 * e + 1] = n;
    etab[4 * e + 2] = R;
    etab[4 * e + 3] = koff;
    auto row_group = [&](int t, int64_t cols) {   // [R][cols] at the expert's padded rows
      int64_t* g = gtab.data() + (static_cast<size_t>(t) * N + e) * 6;
      g[0] = p0;
      g[1] = R;
      g[2] = p0 * cols / 2;
      g[3] = p0 * cols / 16;   // p0 is a multiple of 128: whole scale atoms
      g[4] = 0;
      g[5] = n;
    };
    auto t_group = [&](int t) {   // columns [koff, koff + K256) of a [out_rows][Ksum] matrix
      int64_t* g = gtab.data() + (static_cast<size_t>(t) * N + e) * 6;
      g[0] = p0;
      g[1] = R;
      g[2] = koff / 2;
      g[3] = koff / 64 * 512;   // koff is a multiple of 256: whole scale atoms
      g[4] = K256;
      g[5] = n;
    };
    row_group(0, l);
    t_group(1);
    t_group(2);
    row_group(3, m);
    t_group(4);
    t_group(5);
    ktab[2 * e] = static_cast<int32_t>(koff);
    ktab[2 * e + 1] = static_cast<int32_t>(K256 / 256);
    p0 += ceil_to(n, 128);
    koff += K256;
  }
  int64_t* d_etab = at<int64_t>(ws, L.etab);
  int64_t* d_gtab = at<int64_t>(ws, L.gtab);
  int32_t* d_ktab = at<int32_t>(ws, L.ktab);
  if (cudaMemcpyAsync(d_etab, etab.data(), etab.size() * 8, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(d_gtab, gtab.data(), gtab.size() * 8, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(d_ktab, ktab.data(), ktab.size() * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return LMOE_ERR_CUDA;
  auto gt = [&](int t) { return d_gtab + static_cast<size_t>(t) * N * 6; };

  // every expert's weights with 16 x 16 blocks (current amax per expert and
  // matrix), one grouped launch each: W1 [m][l] and W2 [l][m] for the forward,
  // then W2^T [m][l] and W1^T [l][m] for the dgrads
  if ((st = launch_nvfp4_quantize_ex(W1, LMOE_BF16, m, l, 0, 0, 0, 0, nullptr, at<uint8_t>(ws, L.w1c),
                                     at<uint8_t>(ws, L.w1s), at<float>(ws, L.w1g), tiled2d, part, s, 0, N)) !=
      LMOE_OK)
    return st;
  if ((st = launch_nvfp4_quantize_ex(W2, LMOE_BF16, l, m, 0, 0, 0, 0, nullptr, at<uint8_t>(ws, L.w2c),
                                     at<uint8_t>(ws, L.w2s), at<float>(ws, L.w2g), tiled2d, part, s, 0, N)) !=
      LMOE_OK)
    return st;
  // with 16 x 16 blocks the transposes quantise to the transposed codes and
  // scales, under the same global scales
  if ((st = launch_nvfp4_transpose2d(at<uint8_t>(ws, L.w2c), at<uint8_t>(ws, L.w2s), N, l, m,
                                     at<uint8_t>(ws, L.w2tc), at<uint8_t>(ws, L.w2ts), s)) != LMOE_OK)
    return st;
  if ((st = launch_nvfp4_transpose2d(at<uint8_t>(ws, L.w1c), at<uint8_t>(ws, L.w1s), N, m, l,
                                     at<uint8_t>(ws, L.w1tc), at<uint8_t>(ws, L.w1ts), s)) != LMOE_OK)
    return st;

  // the expert-grouped NVFP4 GEMM over every expert's padded rows
  auto grouped = [&](const void* ac, const uint8_t* as, const float* ag, int ag_grouped, const void* bc,
                     const uint8_t* bs, const float* bg, int64_t cols, int64_t k, void* out, int64_t ld, int f32) {
    Fp4Launch g;
    g.a_codes = ac;
    g.a_sf = as;
    g.a_rows = L.P;
    g.b_codes = bc;
    g.b_sf = bs;
    g.k = k;
    g.cols = static_cast<int>(cols);
    g.groups = N;
    g.offsets = offsets;
    g.padded_offsets = padded_offsets;
    g.in_scale = ag;
    g.in_scale_grouped = ag_grouped;
    g.w_scale = bg;
    g.out = out;
    g.ld_out = ld;
    g.f32_out = f32;
    return L.P > 0 ? fp4_gemm(g, err, s) : LMOE_OK;
  };

  // recomputed forward over all slots: h (fp32), aq (NVFP4 with the static s_a), o (fp32)
  if ((st = grouped(z_codes, z_sf, z_global, 0, at<uint8_t>(ws, L.w1c), at<uint8_t>(ws, L.w1s),
                    at<float>(ws, L.w1g), m, l, at<void>(ws, L.h), m, 1)) != LMOE_OK)
    return st;
  {
    Fp4Launch fq;
    fq.a_codes = z_codes;
    fq.a_sf = z_sf;
    fq.a_rows = L.P;
    fq.b_codes = at<uint8_t>(ws, L.w1c);
    fq.b_sf = at<uint8_t>(ws, L.w1s);
    fq.k = l;
    fq.cols = static_cast<int>(m);
    fq.groups = N;
    fq.offsets = offsets;
    fq.padded_offsets = padded_offsets;
    fq.in_scale = z_global;
    fq.w_scale = at<float>(ws, L.w1g);
    fq.quant_out = 1;
    fq.out_scale = a_global;
    fq.out = at<void>(ws, L.aqc);
    fq.out_sf = at<uint8_t>(ws, L.aqs);
    fq.ld_out = m;
    if (L.P > 0 && (st = fp4_gemm(fq, err, s)) != LMOE_OK) return st;
  }
  if ((st = grouped(at<uint8_t>(ws, L.aqc), at<uint8_t>(ws, L.aqs), a_global, 0, at<uint8_t>(ws, L.w2c),
                    at<uint8_t>(ws, L.w2s), at<float>(ws, L.w2g), l, m, at<void>(ws, L.o), l, 1)) != LMOE_OK)
    return st;

  float* d_o = at<float>(ws, L.d_o);
  float* dh = at<float>(ws, L.dh);
  uint8_t *qac = at<uint8_t>(ws, L.qac), *qas = at<uint8_t>(ws, L.qas);
  float* qag = at<float>(ws, L.qag);
  uint8_t *t1c = at<uint8_t>(ws, L.t1c), *t1s = at<uint8_t>(ws, L.t1s);
  uint8_t *t2c = at<uint8_t>(ws, L.t2c), *t2s = at<uint8_t>(ws, L.t2s);
  float *t1g = at<float>(ws, L.t1g), *t2g = at<float>(ws, L.t2g);
  float* dA = at<float>(ws, L.dA);
  const float* h = at<float>(ws, L.h);
  const float* o = at<float>(ws, L.o);
  const int64_t K256max = ceil_to(L.Rmax, 256);
  const uint32_t T_RHT = LMOE_QX_TRANSPOSE | LMOE_QX_RHT;
  auto quant = [&](int t, const float* in, int64_t cols, uint32_t flags, uint32_t stream0, uint8_t* c, uint8_t* sf,
                   float* g) {
    const bool tr = (flags & LMOE_QX_TRANSPOSE) != 0;
    return launch_nvfp4_quantize_groups(in, LMOE_F32, L.Rmax, cols, flags, rht_signs, seed, stream0, 4, gt(t), N,
                                        tr ? K256max : cols, tr ? L.Ksum : 0, c, sf, g, LMOE_SF_MMA_TILED, part, s);
  };
  float* deq = at<float>(ws, L.deq);
  // every expert's wgrad in one K-batched launch: dW[e] [rows][cols] =
  // A[:, K_e] . B[:, K_e]^T over the expert's K256 columns (experts without
  // rows get a zero gradient)
  auto wgrads = [&](int64_t rows, int64_t cols, void* dw) -> lmoe_status {
    for (int e = 0; e < N; ++e)
      if (counts[e] == 0 &&
          cudaMemsetAsync(static_cast<__nv_bfloat16*>(dw) + e * rows * cols, 0, rows * cols * 2, s) != cudaSuccess)
        return LMOE_ERR_CUDA;
    if (L.Ksum == 0) return LMOE_OK;
    Fp4Launch g;
    g.a_codes = t1c;
    g.a_sf = t1s;
    g.a_rows = rows;
    g.b_codes = t2c;
    g.b_sf = t2s;
    g.k = L.Ksum;
    g.cols = static_cast<int>(cols);
    g.groups = N;
    g.kgroups = d_ktab;
    g.in_scale = t1g;
    g.in_scale_grouped = 1;
    g.w_scale = t2g;
    g.out = dw;
    g.ld_out = cols;
    g.out_group_stride = rows * cols;
    return fp4_gemm(g, err, s);
  };

  // do, dgate
  launch_k(bw_prep_kernel, grid_per_expert(L.Rmax * kBwThreads, N), dim3(kBwThreads), 0, s,
           static_cast<const float*>(dy), o, gate, static_cast<const int64_t*>(d_etab), static_cast<int>(l), d_o,
           dgate, dy_tok, perm_src, offsets, K);
  count_launch();
  // second GEMM, dgrad: dA = SR(do) W2q  (W2^T [m][l] with 16 x 16 blocks)
  if ((st = quant(0, d_o, l, LMOE_QX_SR, 2, qac, qas, qag)) != LMOE_OK) return st;
  if ((st = grouped(qac, qas, qag, 1, at<uint8_t>(ws, L.w2tc), at<uint8_t>(ws, L.w2ts), at<float>(ws, L.w2g), m, l,
                    dA, m, 1)) != LMOE_OK)
    return st;
  // dh
  launch_k(bw_dh_kernel, grid_per_expert(L.Rmax * m, N), dim3(kBwThreads), 0, s, static_cast<const float*>(dA), h,
           static_cast<const int64_t*>(d_etab), static_cast<int>(m), dh);
  count_launch();
  // second GEMM, wgrad: dW2 = SR(RHT(do)^T) RN(RHT(aq)^T)^T  (contraction over the expert's K256 tokens)
  launch_k(bw_dequant_kernel, grid_per_expert(L.Rmax * m / 16, N), dim3(kBwThreads), 0, s,
           static_cast<const uint8_t*>(at<uint8_t>(ws, L.aqc)), static_cast<const uint8_t*>(at<uint8_t>(ws, L.aqs)),
           a_global, static_cast<const int64_t*>(d_etab), static_cast<int>(m), deq);
  count_launch();
  if ((st = quant(1, d_o, l, T_RHT | LMOE_QX_SR, 3, t1c, t1s, t1g)) != LMOE_OK) return st;
  if ((st = quant(2, deq, m, T_RHT, 0, t2c, t2s, t2g)) != LMOE_OK) return st;
  if ((st = wgrads(l, m, dw2)) != LMOE_OK) return st;
  // first GEMM, dgrad: dz = SR(dh) W1q  (W1^T [l][m] with 16 x 16 blocks), at the slot rows
  if ((st = quant(3, dh, m, LMOE_QX_SR, 0, qac, qas, qag)) != LMOE_OK) return st;
  if ((st = grouped(qac, qas, qag, 1, at<uint8_t>(ws, L.w1tc), at<uint8_t>(ws, L.w1ts), at<float>(ws, L.w1g), l, m,
                    dz, l, 0)) != LMOE_OK)
    return st;
  // first GEMM, wgrad: dW1 = SR(RHT(dh)^T) RN(RHT(zq)^T)^T
  launch_k(bw_dequant_kernel, grid_per_expert(L.Rmax * l / 16, N), dim3(kBwThreads), 0, s, z_codes, z_sf, z_global,
           static_cast<const int64_t*>(d_etab), static_cast<int>(l), deq);
  count_launch();
  if ((st = quant(4, dh, m, T_RHT | LMOE_QX_SR, 1, t1c, t1s, t1g)) != LMOE_OK) return st;
  if ((st = quant(5, deq, l, T_RHT, 0, t2c, t2s, t2g)) != LMOE_OK) return st;
  if ((st = wgrads(m, l, dw1)) != LMOE_OK) return st;
  if (o_out && L.P > 0 &&
      cudaMemcpyAsync(o_out, o, static_cast<size_t>(L.P) * l * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return LMOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

}  // namespace lmoe
