// The LatentMoE layer's backward pass with its routed experts trained under
// the NVFP4 recipe (greeksharifa page on the Nemotron 3 whitepaper, sections
// 2.2 "LatentMoE" and 2.4 "NVFP4 Training"; notes.yuuk.io page, section 4).
// The routed experts' GEMMs follow the recipe (lmoe_train_experts.cu); the
// router, the latent projections and the shared experts, which the recipe
// keeps in higher precision, are BF16 tensor-core GEMMs with fp32
// accumulation; every quantiser passes its gradient straight through.
//
//   forward (recomputed): logits = x W_r^T + b, top-K gates, z = x W_dn^T,
//     zq = NVFP4(z) (current amax), slots permuted by expert;
//   dc = dout W_up;  experts: dz per slot, dgate, dW1, dW2, and o;
//   c = sum_k g_k o_k;  dW_up = dout^T c;
//   dsel_k = g_k (dgate_k - sum_j g_j dgate_j) at the chosen experts, 0 elsewhere;
//   dW_r = dsel^T x,  db = sum_t dsel;
//   dz_t = sum_k dz(t,k);  dW_dn = dz^T x;
//   shared expert s: pre = x Ws1_s^T, dWs2_s = dout^T relu(pre)^2,
//     dpre = (dout Ws2_s) * 2 max(pre, 0), dWs1_s = dpre^T x;
//   dx = dsel W_r + dz W_dn + sum_s dpre_s Ws1_s  (dz itself for identity projections).
// Products that contract over the tokens read transposed copies (tokens
// padded with zeros to a multiple of 64); the other transposes are of the
// weights.
#include <cuda_bf16.h>

#include <vector>

#include "gemm_tc.cuh"
#include "lmoe_device.cuh"
#include "lmoe_internal.h"

namespace lmoe {
namespace {

constexpr int kLbThreads = 256;

size_t up256b(size_t b) { return (b + 255) / 256 * 256; }
int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// out[c][r] = in[r][c] as BF16 for r < rows, 0 for rows <= r < pitch
// (in: BF16 or F32, [rows][cols]; out: [cols][pitch]). 32 x 32 tiles through
// shared memory, reads and writes coalesced.
template <typename TI>
__global__ void __launch_bounds__(kLbThreads) transpose_kernel(const TI* __restrict__ in, int64_t rows, int64_t cols,
                                                               int64_t pitch, __nv_bfloat16* __restrict__ out) {
  pdl_begin();
  __shared__ float tile[32][33];
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 32, c0 = static_cast<int64_t>(blockIdx.y) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8 threads
  for (int i = ty; i < 32; i += 8) {
    const int64_t r = r0 + i, c = c0 + tx;
    float v = 0.0f;
    if (r < rows && c < cols) v = static_cast<float>(in[r * cols + c]);
    tile[i][tx] = v;
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int64_t c = c0 + i, r = r0 + tx;
    if (c < cols && r < pitch) out[c * pitch + r] = __float2bfloat16_rn(tile[tx][i]);
  }
}

// y = relu(x)^2 (mode 0) or y = g * 2 max(x, 0) (mode 1), fp32 in, BF16 out.
__global__ void __launch_bounds__(kLbThreads) act_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                                         int64_t n, int mode, __nv_bfloat16* __restrict__ y) {
  pdl_begin();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float r = fmaxf(x[i], 0.0f);
    y[i] = __float2bfloat16_rn(mode == 0 ? r * r : g[i] * (2.0f * r));
  }
}

// y = float(x) (BF16 -> fp32).
__global__ void __launch_bounds__(kLbThreads) widen_kernel(const __nv_bfloat16* __restrict__ x, int64_t n,
                                                            float* __restrict__ y) {
  pdl_begin();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = __bfloat162float(x[i]);
}

// The router's gradient: a warp per token. dgate of slot f sits at its padded
// row; dsel_k = g_k (dgate_k - sum_j g_j dgate_j); dlogits row t (fp32 and
// BF16, [T][N]) is dsel at the chosen experts and 0 elsewhere.
__global__ void __launch_bounds__(kLbThreads) router_grad_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ gates, const int32_t* __restrict__ inv_perm,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ poff, const float* __restrict__ dgate_rows,
    int64_t T, int K, int N, float* __restrict__ dl32, __nv_bfloat16* __restrict__ dl16) {
  pdl_begin();
  const int lane = threadIdx.x & 31;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  for (int n = lane; n < N; n += 32) {
    dl32[t * N + n] = 0.0f;
    dl16[t * N + n] = __float2bfloat16_rn(0.0f);
  }
  __syncwarp();
  float g = 0.0f, dg = 0.0f;
  int e = -1;
  if (lane < K) {
    const int64_t f = t * K + lane;
    e = __ldg(idx + f);
    if (e >= 0 && e < N) {
      g = __ldg(gates + f);
      const int64_t row = static_cast<int64_t>(__ldg(inv_perm + f)) - __ldg(offsets + e) + __ldg(poff + e);
      dg = __ldg(dgate_rows + row);
    } else {
      e = -1;
    }
  }
  float sgd = g * dg;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sgd += __shfl_xor_sync(0xffffffffu, sgd, off);
  __syncwarp();
  if (e >= 0) {
    const float v = g * (dg - sgd);
    dl32[t * N + e] = v;
    dl16[t * N + e] = __float2bfloat16_rn(v);
  }
}

// db[n] = sum over t of dl[t][n], in t order (fp32).
__global__ void __launch_bounds__(kLbThreads) colsum_kernel(const float* __restrict__ dl, int64_t T, int N,
                                                            float* __restrict__ db) {
  pdl_begin();
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  float s = 0.0f;
  for (int64_t t = 0; t < T; ++t) s += dl[t * N + n];
  db[n] = s;
}

struct LbLayout {
  size_t err, logits, idx, gates, z, zq, zsf, zgs, qpart, offs, poff, psrc, iperm, scratch, pgate, zp, zpsf, dc,
      dzr, dgate, o, c, dzt, dl32, dl16, dlT, xT, doT, cT, dzT, wupT, wrT, wdnT, pre, hs, hsT, tmp, dpre, dpreT, ws2T,
      ws1T, ex, total;
  int64_t P, T64;
};

LbLayout lb_layout(const lmoe_config* c) {
  LbLayout L = {};
  const int64_t T = c->T, d = c->d, l = c->l, N = c->N, K = c->K;
  const int64_t Sms = static_cast<int64_t>(c->n_shared) * c->m_shared;
  const bool ident = (c->flags & LMOE_FLAG_IDENTITY_PROJ) != 0;
  L.P = lmoe_padded_rows(c);
  L.T64 = round_up(T > 0 ? T : 1, 64);
  size_t off = 0;
  auto take = [&](size_t b) {
    const size_t o = off;
    off += up256b(b);
    return o;
  };
  L.err = take(256);
  L.logits = take(T * N * 4);
  L.idx = take(T * K * 4);
  L.gates = take(T * K * 4);
  L.z = ident ? 0 : take(T * l * 2);
  L.zq = take(T * l / 2);
  L.zsf = take(T * l / 16);
  L.zgs = take(16);
  L.qpart = take(static_cast<size_t>(nvfp4_partials(T * l)) * 4);
  L.offs = take((N + 1) * 4);
  L.poff = take((N + 1) * 4);
  L.psrc = take(T * K * 4);
  L.iperm = take(T * K * 4);
  L.scratch = take(static_cast<size_t>(permute_chunks(T * K) + 1) * N * 4);
  L.pgate = take(L.P * 4);
  L.zp = take(L.P * l / 2);
  L.zpsf = take(L.P * l / 16);
  L.dc = take(T * l * 4);
  L.dzr = take(L.P * l * 2);
  L.dgate = take(L.P * 4);
  L.o = take(L.P * l * 4);
  L.c = take(T * l * 4);
  L.dzt = take(T * l * 2);
  L.dl32 = take(T * N * 4);
  L.dl16 = take(T * N * 2);
  L.dlT = take(N * L.T64 * 2);
  L.xT = take(d * L.T64 * 2);
  L.doT = take(d * L.T64 * 2);
  L.cT = take(l * L.T64 * 2);
  L.dzT = take(l * L.T64 * 2);
  L.wupT = ident ? 0 : take(l * d * 2);
  L.wrT = take(d * N * 2);
  L.wdnT = ident ? 0 : take(d * l * 2);
  if (Sms > 0) {
    L.pre = take(T * Sms * 4);
    L.hs = take(T * Sms * 2);
    L.hsT = take(Sms * L.T64 * 2);
    L.tmp = take(T * Sms * 4);
    L.dpre = take(T * Sms * 2);
    L.dpreT = take(Sms * L.T64 * 2);
    L.ws2T = take(Sms * d * 2);
    L.ws1T = take(d * Sms * 2);
  }
  L.ex = take(expert_backward_ws_bound(c));   // any routing of the T tokens
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

unsigned grid_of(int64_t items) {
  const int64_t sms = device_sm_count();
  int64_t b = (items + kLbThreads - 1) / kLbThreads;
  if (b > sms * 8) b = sms * 8;
  return static_cast<unsigned>(b < 1 ? 1 : b);
}

template <typename TI>
lmoe_status transpose(const TI* in, int64_t rows, int64_t cols, int64_t pitch, void* out, cudaStream_t s) {
  if (rows == 0 && pitch == 0) return LMOE_OK;
  const int64_t gr = (pitch + 31) / 32, gc = (cols + 31) / 32;
  if (gr > 0x7fffffff || gc > 65535) return LMOE_ERR_UNSUPPORTED;
  launch_k(transpose_kernel<TI>, dim3(static_cast<unsigned>(gr), static_cast<unsigned>(gc)), dim3(kLbThreads), 0, s, in,
           rows, cols, pitch, static_cast<__nv_bfloat16*>(out));
  count_launch();
  return LMOE_OK;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace lmoe

using namespace lmoe;

extern "C" {

size_t lmoe_backward_nvfp4_workspace(const lmoe_config* cfg) {
  if (!cfg || cfg->T < 0 || cfg->N <= 0 || cfg->K <= 0) return 0;
  return lb_layout(cfg).total;
}

lmoe_status lmoe_backward_nvfp4(const lmoe_config* cfg, const lmoe_weights* w, const void* x, const void* dout,
                                const float* a_global, uint64_t seed, uint32_t rht_signs, const lmoe_grads* g,
                                void* ws, size_t ws_bytes, void* stream) {
  if (!cfg || !w || !x || !dout || !a_global || !g) return LMOE_ERR_INVALID_ARG;
  const int64_t T = cfg->T, d = cfg->d, l = cfg->l, N = cfg->N, K = cfg->K, m = cfg->m;
  const int S = cfg->n_shared;
  const int64_t ms = cfg->m_shared, Sms = static_cast<int64_t>(S) * ms;
  const bool ident = (cfg->flags & LMOE_FLAG_IDENTITY_PROJ) != 0;
  if (T < 0 || d <= 0 || l <= 0 || N <= 0 || K <= 0 || K > N || m <= 0 || S < 0) return LMOE_ERR_INVALID_ARG;
  if (cfg->act != LMOE_BF16 || cfg->expert != LMOE_BF16 || (cfg->flags & LMOE_FLAG_SHARED_FP8))
    return LMOE_ERR_UNSUPPORTED;
  if (K > 32 || N > 1024 || N % 8 || d % 64 || l % 256 || m % 256 || (S && ms % 64)) return LMOE_ERR_UNSUPPORTED;
  if (ident && l != d) return LMOE_ERR_INVALID_ARG;
  if (!w->w_router || !w->w1 || !w->w2 || ident != (w->w_down == nullptr) || ident != (w->w_up == nullptr) ||
      (S && (!w->ws1 || !w->ws2)))
    return LMOE_ERR_INVALID_ARG;
  if (!g->dx || !g->dw_router || !g->dw1 || !g->dw2 || (!ident && (!g->dw_down || !g->dw_up)) ||
      (w->router_bias && !g->drouter_bias) || (S && (!g->dws1 || !g->dws2)))
    return LMOE_ERR_INVALID_ARG;
  if (!al16(x) || !al16(dout) || !al16(g->dx) || !al16(g->dw_router) || !al16(g->dw1) || !al16(g->dw2))
    return LMOE_ERR_INVALID_ARG;
  const LbLayout L = lb_layout(cfg);
  if (!ws || ws_bytes < L.total) return LMOE_ERR_WORKSPACE;
  if (T == 0) return LMOE_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* err = at<uint32_t>(ws, L.err);
  lmoe_status st = LMOE_OK;
  const int64_t T64 = L.T64;
  auto ok = [&](lmoe_status v) { return (st = v) == LMOE_OK; };

  // ---- forward pieces: routing, z, NVFP4 z rows in the experts' padded layout ----
  float* logits = at<float>(ws, L.logits);
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* gates = at<float>(ws, L.gates);
  if (!ok(dense_bf16(x, T, w->w_router, static_cast<int>(N), d, logits, N, EPI_F32_BIAS, w->router_bias, nullptr, 0,
                     nullptr, err, s)))
    return st;
  // gates from exact logits: the experts' stochastic quantisers read gate * dy
  if (!ok(launch_topk(logits, T, static_cast<int>(N), static_cast<int>(K), idx, gates, x, w->w_router,
                      w->router_bias, static_cast<int>(d), LMOE_BF16, err, s, 1)))
    return st;
  const void* z = x;
  if (!ident) {
    if (!ok(dense_bf16(x, T, w->w_down, static_cast<int>(l), d, at<void>(ws, L.z), l, EPI_BF16, nullptr, nullptr, 0,
                       nullptr, err, s)))
      return st;
    z = at<void>(ws, L.z);
  }
  float* zgs = at<float>(ws, L.zgs);
  if (!ok(launch_nvfp4_quantize(z, LMOE_BF16, T, l, nullptr, at<uint8_t>(ws, L.zq), at<uint8_t>(ws, L.zsf), zgs,
                                LMOE_SF_ROWMAJOR, at<float>(ws, L.qpart), nvfp4_partials(T * l), err, s)))
    return st;
  int32_t* offs = at<int32_t>(ws, L.offs);
  int32_t* poff = at<int32_t>(ws, L.poff);
  int32_t* iperm = at<int32_t>(ws, L.iperm);
  int32_t* psrc = at<int32_t>(ws, L.psrc);
  float* pgate = at<float>(ws, L.pgate);
  if (!ok(launch_permute(idx, T, static_cast<int>(K), static_cast<int>(N), offs, psrc, iperm, poff,
                         at<int32_t>(ws, L.scratch), gates, pgate, err, s)))
    return st;
  if (!ok(launch_gather(idx, psrc, offs, poff, T * K, static_cast<int>(K), at<uint8_t>(ws, L.zq), l / 2,
                        at<uint8_t>(ws, L.zp), at<uint8_t>(ws, L.zsf), at<uint8_t>(ws, L.zpsf), static_cast<int>(N), s)))
    return st;
  // upstream gradient of the combine: dc = dout W_up (fp32: the experts' stochastic quantisers read it)
  float* dc = at<float>(ws, L.dc);
  if (!ident) {
    if (!ok(transpose(static_cast<const __nv_bfloat16*>(w->w_up), d, l, d, at<void>(ws, L.wupT), s))) return st;
    if (!ok(dense_bf16(dout, T, at<void>(ws, L.wupT), static_cast<int>(l), d, dc, l, EPI_F32_BIAS, nullptr, nullptr, 0,
                       nullptr, err, s)))
      return st;
  } else {
    launch_k(widen_kernel, dim3(grid_of(T * l)), dim3(kLbThreads), 0, s, static_cast<const __nv_bfloat16*>(dout),
             T * l, dc);
    count_launch();
  }
  // each slot row's upstream gradient is dc of its token (fp32): the experts'
  // backward reads it through the permutation, no per-slot copy

  // ---- the routed experts (NVFP4 recipe); they need their row counts on the host ----
  std::vector<int32_t> off_h(N + 1);
  if (cudaMemcpyAsync(off_h.data(), offs, (N + 1) * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return LMOE_ERR_CUDA;
  std::vector<int32_t> counts(N);
  for (int64_t e = 0; e < N; ++e) counts[e] = off_h[e + 1] - off_h[e];
  void* ex = at<void>(ws, L.ex);
  float* o = at<float>(ws, L.o);
  float* dgate = at<float>(ws, L.dgate);
  __nv_bfloat16* dzr = at<__nv_bfloat16>(ws, L.dzr);
  if (!ok(expert_backward_core(cfg, counts.data(), offs, poff, at<uint8_t>(ws, L.zp), at<uint8_t>(ws, L.zpsf), zgs,
                               w->w1, w->w2, a_global, pgate, nullptr, seed, rht_signs, dzr, dgate, g->dw1, g->dw2,
                               ex, o, err, s, dc, psrc, static_cast<int>(K))))
    return st;

  // c = sum_k g_k o_k (fp32), dz_t = sum_k dz(t, k) (BF16)
  float* c = at<float>(ws, L.c);
  __nv_bfloat16* dzt = at<__nv_bfloat16>(ws, L.dzt);
  if (!ok(launch_combine(o, LMOE_F32, idx, iperm, offs, poff, gates, nullptr, c, T, static_cast<int>(K),
                         static_cast<int>(N), static_cast<int>(l), s)))
    return st;
  if (!ok(launch_combine(dzr, LMOE_BF16, idx, iperm, offs, poff, nullptr, nullptr, dzt, T, static_cast<int>(K),
                         static_cast<int>(N), static_cast<int>(l), s)))
    return st;

  // ---- router ----
  float* dl32 = at<float>(ws, L.dl32);
  __nv_bfloat16* dl16 = at<__nv_bfloat16>(ws, L.dl16);
  launch_k(router_grad_kernel, dim3(static_cast<unsigned>((T * 32 + kLbThreads - 1) / kLbThreads)), dim3(kLbThreads),
           0, s, static_cast<const int32_t*>(idx), static_cast<const float*>(gates), static_cast<const int32_t*>(iperm),
           static_cast<const int32_t*>(offs), static_cast<const int32_t*>(poff), static_cast<const float*>(dgate), T,
           static_cast<int>(K), static_cast<int>(N), dl32, dl16);
  count_launch();
  if (w->router_bias) {
    launch_k(colsum_kernel, dim3(static_cast<unsigned>((N + kLbThreads - 1) / kLbThreads)), dim3(kLbThreads), 0, s,
             static_cast<const float*>(dl32), T, static_cast<int>(N), g->drouter_bias);
    count_launch();
  }

  // ---- products over the tokens: transposed copies, tokens padded to T64 ----
  void* xT = at<void>(ws, L.xT);
  void* doT = at<void>(ws, L.doT);
  void* dlT = at<void>(ws, L.dlT);
  if (!ok(transpose(static_cast<const __nv_bfloat16*>(x), T, d, T64, xT, s))) return st;
  if (!ok(transpose(dl16, T, N, T64, dlT, s))) return st;
  if (!ok(dense_bf16(dlT, N, xT, static_cast<int>(d), T64, g->dw_router, d, EPI_BF16, nullptr, nullptr, 0, nullptr, err,
                     s)))
    return st;
  if (!ident || S > 0)
    if (!ok(transpose(static_cast<const __nv_bfloat16*>(dout), T, d, T64, doT, s))) return st;
  if (!ident) {
    void* cT = at<void>(ws, L.cT);
    void* dzT = at<void>(ws, L.dzT);
    if (!ok(transpose(c, T, l, T64, cT, s))) return st;
    if (!ok(dense_bf16(doT, d, cT, static_cast<int>(l), T64, g->dw_up, l, EPI_BF16, nullptr, nullptr, 0, nullptr, err,
                       s)))
      return st;
    if (!ok(transpose(dzt, T, l, T64, dzT, s))) return st;
    if (!ok(dense_bf16(dzT, l, xT, static_cast<int>(d), T64, g->dw_down, d, EPI_BF16, nullptr, nullptr, 0, nullptr,
                       err, s)))
      return st;
  }

  // ---- dx = dsel W_r + dz W_dn (dz itself with identity projections) ----
  void* wrT = at<void>(ws, L.wrT);
  if (!ok(transpose(static_cast<const __nv_bfloat16*>(w->w_router), N, d, N, wrT, s))) return st;
  if (!ident) {
    void* wdnT = at<void>(ws, L.wdnT);
    if (!ok(transpose(static_cast<const __nv_bfloat16*>(w->w_down), l, d, l, wdnT, s))) return st;
    if (!ok(dense_bf16(dzt, T, wdnT, static_cast<int>(d), l, g->dx, d, EPI_BF16, nullptr, nullptr, 0, nullptr, err, s)))
      return st;
    if (!ok(dense_bf16(dl16, T, wrT, static_cast<int>(d), N, g->dx, d, EPI_ADD_RES, nullptr, g->dx, d, nullptr, err, s)))
      return st;
  } else {
    if (!ok(dense_bf16(dl16, T, wrT, static_cast<int>(d), N, g->dx, d, EPI_ADD_RES, nullptr, dzt, d, nullptr, err, s)))
      return st;
  }

  // ---- shared experts (BF16, on the d-dim x) ----
  if (S > 0) {
    float* pre = at<float>(ws, L.pre);
    __nv_bfloat16* hs = at<__nv_bfloat16>(ws, L.hs);
    float* tmp = at<float>(ws, L.tmp);
    __nv_bfloat16* dpre = at<__nv_bfloat16>(ws, L.dpre);
    void* hsT = at<void>(ws, L.hsT);
    void* dpreT = at<void>(ws, L.dpreT);
    uint8_t* ws2T = at<uint8_t>(ws, L.ws2T);
    void* ws1T = at<void>(ws, L.ws1T);
    if (!ok(dense_bf16(x, T, w->ws1, static_cast<int>(Sms), d, pre, Sms, EPI_F32_BIAS, nullptr, nullptr, 0, nullptr,
                       err, s)))
      return st;
    launch_k(act_kernel, dim3(grid_of(T * Sms)), dim3(kLbThreads), 0, s, static_cast<const float*>(pre),
             static_cast<const float*>(nullptr), T * Sms, 0, hs);
    count_launch();
    for (int sh = 0; sh < S; ++sh)   // Ws2_s [d][ms] -> [ms][d], stacked over s
      if (!ok(transpose(static_cast<const __nv_bfloat16*>(w->ws2) + sh * d * ms, d, ms, d, ws2T + sh * ms * d * 2, s)))
        return st;
    if (!ok(dense_bf16(dout, T, ws2T, static_cast<int>(Sms), d, tmp, Sms, EPI_F32_BIAS, nullptr, nullptr, 0, nullptr,
                       err, s)))
      return st;
    launch_k(act_kernel, dim3(grid_of(T * Sms)), dim3(kLbThreads), 0, s, static_cast<const float*>(pre),
             static_cast<const float*>(tmp), T * Sms, 1, dpre);
    count_launch();
    if (!ok(transpose(hs, T, Sms, T64, hsT, s))) return st;
    for (int sh = 0; sh < S; ++sh)
      if (!ok(dense_bf16(doT, d, static_cast<const __nv_bfloat16*>(hsT) + sh * ms * T64, static_cast<int>(ms), T64,
                         static_cast<__nv_bfloat16*>(g->dws2) + sh * d * ms, ms, EPI_BF16, nullptr, nullptr, 0,
                         nullptr, err, s)))
        return st;
    if (!ok(transpose(dpre, T, Sms, T64, dpreT, s))) return st;
    if (!ok(dense_bf16(dpreT, Sms, xT, static_cast<int>(d), T64, g->dws1, d, EPI_BF16, nullptr, nullptr, 0, nullptr,
                       err, s)))
      return st;
    if (!ok(transpose(static_cast<const __nv_bfloat16*>(w->ws1), Sms, d, Sms, ws1T, s))) return st;
    if (!ok(dense_bf16(dpre, T, ws1T, static_cast<int>(d), Sms, g->dx, d, EPI_ADD_RES, nullptr, g->dx, d, nullptr,
                       err, s)))
      return st;
  }
  return cudaGetLastError() == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}

}  // extern "C"
