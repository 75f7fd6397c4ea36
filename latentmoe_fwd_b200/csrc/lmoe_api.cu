// C ABI of the LatentMoE layer forward: argument checks, workspace carving and
// the launch sequence of each entry point. Every launch is asynchronous on the
// caller's stream; nothing here allocates device memory.
#include <atomic>
#include <cstring>
#include <functional>

#include "gemm_tc.cuh"
#include "lmoe_internal.h"

namespace lmoe {

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int device_sm_count() {
  static std::atomic<int> cache[64];   // 0 = not queried yet
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev >= 0 && dev < 64;
  int n = cached ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (cached) cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

namespace {

constexpr size_t kAlign = 256;
size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

size_t act_bytes(const lmoe_config* c) { return c->act == LMOE_F32 ? 4 : 2; }

bool identity(const lmoe_config* c) { return (c->flags & LMOE_FLAG_IDENTITY_PROJ) != 0; }

// A host thread's second stream on a device (highest priority) with the two
// events that fork work onto it and join it back, created on first use and
// kept for the thread's life. Per thread, so that concurrent callers never
// record one another's events.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

bool side_stream(SideStream* out) {
  thread_local SideStream per_device[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  SideStream& ss = per_device[dev];
  if (!ss.stream) {
    int lo = 0, hi = 0;
    SideStream made;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess ||
        cudaStreamCreateWithPriority(&made.stream, cudaStreamNonBlocking, hi) != cudaSuccess)
      return false;
    if (cudaEventCreateWithFlags(&made.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&made.join, cudaEventDisableTiming) != cudaSuccess) {
      if (made.fork) cudaEventDestroy(made.fork);
      cudaStreamDestroy(made.stream);
      return false;
    }
    ss = made;
  }
  *out = ss;
  return true;
}

int64_t padded_rows(const lmoe_config* c) {
  const int64_t slots = c->T * c->K;
  const int64_t nonempty = slots < c->N ? slots : c->N;
  return (slots + 127 * nonempty + 127) / 128 * 128;
}

lmoe_status check_config(const lmoe_config* c) {
  if (!c) return LMOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->T > (int64_t(1) << 31) / 64) return LMOE_ERR_INVALID_ARG;
  if (c->d <= 0 || c->l <= 0 || c->N <= 0 || c->K <= 0 || c->m <= 0) return LMOE_ERR_INVALID_ARG;
  if (c->K > c->N) return LMOE_ERR_INVALID_ARG;
  if (c->K > 32 || c->N > 1024) return LMOE_ERR_UNSUPPORTED;
  if (c->n_shared < 0 || (c->n_shared > 0 && c->m_shared <= 0)) return LMOE_ERR_INVALID_ARG;
  if (c->d % 8 || c->l % 8 || c->m % 8 || (c->n_shared && c->m_shared % 8)) return LMOE_ERR_INVALID_ARG;
  if (identity(c) && c->l != c->d) return LMOE_ERR_INVALID_ARG;
  if (c->act != LMOE_F32 && c->act != LMOE_BF16) return LMOE_ERR_UNSUPPORTED;
  if (c->act == LMOE_F32 && c->expert != LMOE_F32) return LMOE_ERR_UNSUPPORTED;
  if (c->act == LMOE_BF16 && c->expert != LMOE_BF16 && c->expert != LMOE_NVFP4) return LMOE_ERR_UNSUPPORTED;
  if (c->act == LMOE_BF16 && c->n_shared > 0 && c->m_shared % 64) return LMOE_ERR_UNSUPPORTED;
  if (c->expert == LMOE_NVFP4 && (c->l % 256 || c->m % 256)) return LMOE_ERR_UNSUPPORTED;
  if (c->flags & LMOE_FLAG_SHARED_FP8) {
    if (c->n_shared <= 0) return LMOE_ERR_INVALID_ARG;
    if (c->act != LMOE_BF16 || c->d % 16 || c->m_shared % 128) return LMOE_ERR_UNSUPPORTED;
  }
  return LMOE_OK;
}

bool shared_fp8(const lmoe_config* c) { return (c->flags & LMOE_FLAG_SHARED_FP8) != 0 && c->n_shared > 0; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Weight-major (swap) tiles are used up to this many tokens.
constexpr int64_t kSwapMaxTokens = 64;
// Split-K of the weight-major dense GEMMs: at most this many splits.
constexpr int kMaxSplits = 32;

int64_t max_dense_cols(const lmoe_config* c, int op) {
  int64_t m = c->N;
  if (op == LMOE_OP_FORWARD) {
    m = m > c->l ? m : c->l;
    m = m > c->d ? m : c->d;
    const int64_t sh = static_cast<int64_t>(c->n_shared) * c->m_shared;
    m = m > sh ? m : sh;
  }
  return m;
}

int64_t splitk_floats(const lmoe_config* c, int op) { return c->T * max_dense_cols(c, op) * kMaxSplits; }

// Workspace layout (byte offsets; region sizes 0 when unused).
struct Layout {
  size_t splitk = 0;        // fp32 split-K partial sums of the weight-major dense GEMMs (T <= 64)
  size_t rsplit = 0;        // fp32 split-K partial sums of the token-major router GEMM (few tiles)
  size_t err = 0, logits = 0, idx = 0, w = 0, z = 0, z_gs = 0, partials = 0, xq = 0,
         offsets = 0, poff = 0, perm_src = 0, inv_perm = 0, slot_row = 0, scratch = 0, gate = 0, zp = 0,
         zp_sf = 0, a = 0, a_sf = 0, y = 0, c = 0, hs = 0, ys = 0, total = 0;
};

int tokmajor_splits(int64_t rows, int cols, int64_t k);

Layout layout(const lmoe_config* c, int op) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += up(bytes);
    return o;
  };
  const int64_t T = c->T, K = c->K, N = c->N;
  const int64_t P = padded_rows(c);
  const size_t ab = act_bytes(c);
  const bool fp4 = c->expert == LMOE_NVFP4;
  L.err = take(256);
  if ((op == LMOE_OP_ROUTE || op == LMOE_OP_FORWARD) && T <= kSwapMaxTokens)
    L.splitk = take(splitk_floats(c, op) * 4);
  if ((op == LMOE_OP_ROUTE || op == LMOE_OP_FORWARD) && T > kSwapMaxTokens && c->act != LMOE_F32) {
    const int sp = tokmajor_splits(T, static_cast<int>(N), c->d);
    if (sp > 1) L.rsplit = take(static_cast<size_t>(T) * N * sp * 4);
  }
  if (op == LMOE_OP_ROUTE) {
    L.logits = take(T * N * 4);
  } else if (op == LMOE_OP_PERMUTE) {
    L.scratch = take(static_cast<size_t>(permute_chunks(T * K) + 1) * N * 4);
  } else if (op == LMOE_OP_EXPERT_FFN) {
    L.a = take(P * c->m * (fp4 ? 1 : ab) / (fp4 ? 2 : 1));
    if (fp4) L.a_sf = take(P * c->m / 16);
  } else if (op == LMOE_OP_NVFP4_QUANTIZE || op == LMOE_OP_FP8_QUANTIZE) {
    L.partials = take(nvfp4_partials(T * c->l) * 4);
  } else if (op == LMOE_OP_FORWARD) {
    L.logits = take(T * N * 4);
    L.idx = take(T * K * 4);
    L.w = take(T * K * 4);
    if (!identity(c)) L.z = take(T * c->l * ab);
    if (fp4) {
      L.z_gs = take(16);
      L.partials = take(nvfp4_partials(T * c->l) * 4);
    }
    L.offsets = take((N + 1) * 4);
    L.poff = take((N + 1) * 4);
    L.perm_src = take(T * K * 4);
    L.inv_perm = take(T * K * 4);
    L.slot_row = take(T * K * 4);
    L.scratch = take(static_cast<size_t>(permute_chunks(T * K) + 1) * N * 4);
    L.gate = take(P * 4);
    if (fp4) {
      L.zp = take(P * c->l / 2);
      L.zp_sf = take(P * c->l / 16);
      L.a = take(P * c->m / 2);
      L.a_sf = take(P * c->m / 16);
    } else {
      L.zp = take(P * c->l * ab);
      L.a = take(P * c->m * ab);
    }
    L.y = take(P * c->l * ab);
    L.c = take(T * c->l * ab);
    if (c->n_shared) {
      L.hs = take(T * static_cast<int64_t>(c->n_shared) * c->m_shared * ab);   // E4M3 codes with FP8 shared experts
      L.ys = take(T * c->d * ab);
      if (shared_fp8(c)) L.xq = take(T * c->d);
    }
  }
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

uint32_t* err_word(void* ws) { return static_cast<uint32_t*>(ws); }

// Token-count threshold below which GEMMs put the weights on the MMA's M side.
int swap_bn(int64_t T) { return T <= 32 ? 32 : (T <= 64 ? 64 : 0); }

int normal_bn(int cols) { return cols >= 256 ? 256 : cols > 64 ? 128 : cols > 32 ? 64 : 32; }

int kblocks(int64_t k) { return static_cast<int>((k + 63) / 64); }

// Splits for a weight-major GEMM with `tiles` output tiles and `kb` K blocks:
// as many as fit in one wave of the GPU (a second, partial wave would double
// the time of a weight-streaming GEMM), at least two K blocks per split,
// within the buffer.
int choose_splits(int64_t tiles, int kb, float* partial) {
  if (!partial) return 1;
  const int sms = device_sm_count();
  int sp = static_cast<int>(sms / tiles);
  if (sp > kb / 2) sp = kb / 2;
  if (sp > kMaxSplits) sp = kMaxSplits;
  return sp > 1 ? sp : 1;
}

// Split-K of a token-major dense GEMM whose 128 x BN tiles fill less than half
// the GPU (the router at a few thousand tokens): splits to fill one wave, at
// least two K blocks each, at most 8.
int tokmajor_splits(int64_t rows, int cols, int64_t k) {
  const int bn = normal_bn(cols);
  const int64_t tiles = ((rows + 127) / 128) * ((cols + bn - 1) / bn);
  const int sms = device_sm_count();
  if (tiles * 2 > sms) return 1;
  int sp = static_cast<int>(sms / tiles);
  const int kb = kblocks(k);
  if (sp > kb / 2) sp = kb / 2;
  if (sp > 8) sp = 8;
  return sp > 1 ? sp : 1;
}

}  // namespace

// out[rows, cols] = epi(x[rows, k] . W[cols, k]^T) with BF16 operands.
lmoe_status dense_bf16(const void* x, int64_t rows, const void* w, int cols, int64_t k, void* out,
                       int64_t ld_out, int epi, const float* bias, const void* residual, int64_t ld_res,
                       float* partial, uint32_t* err, cudaStream_t s) {
  if (rows == 0) return LMOE_OK;
  TcLaunch L;
  const int sbn = swap_bn(rows);
  const TcOperand act{x, k, rows, 1};
  const TcOperand wt{w, k, cols, 1};
  L.rows = static_cast<int>(rows);
  L.cols = cols;
  L.kblocks[0] = kblocks(k);
  if (sbn) {
    L.swap = 1;
    L.bn = sbn;
    L.a[0] = wt;
    L.b[0] = act;
    L.max_tiles = (cols + 127) / 128;
    L.ksplit = choose_splits(L.max_tiles, L.kblocks[0], partial);
    L.partial = partial;
  } else {
    L.bn = normal_bn(cols);
    L.a[0] = act;
    L.b[0] = wt;
    L.max_tiles = ((rows + 127) / 128) * ((cols + L.bn - 1) / L.bn);
    if (partial) {   // a buffer of rows * cols * tokmajor_splits() floats
      L.ksplit = tokmajor_splits(rows, cols, k);
      L.partial = partial;
    }
  }
  L.out = out;
  L.ld_out = ld_out;
  L.epi = epi;
  L.bias = bias;
  L.residual = residual;
  L.ld_res = ld_res;
  return tc_gemm(L, err, s);
}

namespace {

// out[rows, cols] = epi(x[rows, k] . W^T) with E4M3 operands; W is [cols][k],
// or [k / wgroup][cols][wgroup] (the K axis split over a stack of matrices)
// when wgroup > 0. epi: EPI_SQRELU_Q8 (E4M3 out) or EPI_SCALE (BF16 out).
lmoe_status dense_fp8(const void* x, int64_t rows, const void* w, int cols, int64_t k, int wgroup, void* out,
                      int64_t ld_out, int epi, const float* scale_a, const float* scale_w, const float* out_scale,
                      float* partial, uint32_t* err, cudaStream_t s) {
  if (rows == 0) return LMOE_OK;
  TcLaunch L;
  const int sbn = swap_bn(rows);
  TcOperand act{x, k, rows, 1};
  act.elem = 1;
  TcOperand wt{w, wgroup ? wgroup : k, cols, wgroup ? k / wgroup : 1};
  wt.elem = 1;
  L.fp8 = 1;
  L.rows = static_cast<int>(rows);
  L.cols = cols;
  L.kblocks[0] = static_cast<int>((k + 127) / 128);
  if (sbn) {
    L.swap = 1;
    L.bn = sbn;
    L.a[0] = wt;
    L.b[0] = act;
    L.a_kgroup[0] = wgroup;
    L.max_tiles = (cols + 127) / 128;
    L.ksplit = choose_splits(L.max_tiles, L.kblocks[0], partial);
    L.partial = partial;
  } else {
    L.bn = normal_bn(cols);
    L.a[0] = act;
    L.b[0] = wt;
    L.b_kgroup[0] = wgroup;
    L.max_tiles = ((rows + 127) / 128) * ((cols + L.bn - 1) / L.bn);
  }
  L.out = out;
  L.ld_out = ld_out;
  L.epi = epi;
  L.scale_a = scale_a;
  L.scale_w = scale_w;
  L.out_scale = out_scale;
  return tc_gemm(L, err, s);
}

// The shared experts in FP8: xq = E4M3(x / s_x); hs = E4M3(relu(xq Ws1^T * s_x
// s_w1)^2 / s_h) over all S experts at once; ys = hs [Ws2_1 .. Ws2_S]^T * s_h
// s_w2 in BF16 (added to the layer output by the combine or the up-projection).
lmoe_status shared_experts_fp8(const lmoe_config* cfg, const lmoe_weights* w, const void* x, uint8_t* xq,
                               uint8_t* hq, void* ys, float* partial, uint32_t* err, cudaStream_t s) {
  const int64_t T = cfg->T;
  const int S = cfg->n_shared, ms = cfg->m_shared, d = cfg->d;
  lmoe_status st = launch_fp8_quantize(x, LMOE_BF16, T, d, w->shared_x_scale, xq, nullptr, nullptr, 0, s);
  if (st != LMOE_OK) return st;
  st = dense_fp8(xq, T, w->ws1, S * ms, d, 0, hq, static_cast<int64_t>(S) * ms, EPI_SQRELU_Q8, w->shared_x_scale,
                 w->ws1_scale, w->shared_h_scale, partial, err, s);
  if (st != LMOE_OK) return st;
  return dense_fp8(hq, T, w->ws2, d, static_cast<int64_t>(S) * ms, ms, ys, d, EPI_SCALE, w->shared_h_scale,
                   w->ws2_scale, nullptr, partial, err, s);
}

}  // namespace
}  // namespace lmoe

using namespace lmoe;

extern "C" {

const char* lmoe_status_string(lmoe_status s) {
  switch (s) {
    case LMOE_OK: return "ok";
    case LMOE_ERR_INVALID_ARG: return "invalid argument";
    case LMOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case LMOE_ERR_WORKSPACE: return "workspace missing or too small";
    case LMOE_ERR_CUDA: return "CUDA error";
    case LMOE_ERR_DEVICE_TIMEOUT: return "device pipeline wait timed out";
    case LMOE_ERR_DEVICE_BOUNDS: return "device index out of range";
  }
  return "unknown status";
}

uint64_t lmoe_kernel_launch_count(void) { return g_launches.load(); }

lmoe_status lmoe_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t limit_cycles, void* stream) {
  if (!ws || ws_bytes < 256) return LMOE_ERR_WORKSPACE;
  if (limit_cycles == 0 || limit_cycles > static_cast<uint64_t>(kWaitLimitCycles)) return LMOE_ERR_INVALID_ARG;
  return launch_selftest_wait(err_word(ws), static_cast<long long>(limit_cycles), static_cast<cudaStream_t>(stream));
}

size_t lmoe_workspace_size(const lmoe_config* cfg, int op) {
  if (op == LMOE_OP_NVFP4_QUANTIZE || op == LMOE_OP_FP8_QUANTIZE) {
    if (!cfg || cfg->T < 0 || cfg->l <= 0) return 0;
    return layout(cfg, op).total;
  }
  if (check_config(cfg) != LMOE_OK) return 0;
  if (op == LMOE_OP_COMBINE) return 0;
  if (op < LMOE_OP_ROUTE || op > LMOE_OP_NVFP4_QUANTIZE) return 0;
  return layout(cfg, op).total;
}

int64_t lmoe_padded_rows(const lmoe_config* cfg) {
  if (check_config(cfg) != LMOE_OK) return 0;
  return padded_rows(cfg);
}

lmoe_status lmoe_read_device_error(void* ws, void* stream, uint32_t* info) {
  if (!ws) return LMOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return LMOE_ERR_CUDA;
  // read and clear on the caller's stream, so the clear is ordered before any
  // kernel the caller launches on it afterwards (a plain cudaMemset runs on the
  // legacy stream, which a non-blocking stream does not wait for)
  uint32_t w[2] = {0, 0};
  if (cudaMemcpyAsync(w, ws, sizeof(w), cudaMemcpyDeviceToHost, s) != cudaSuccess) return LMOE_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(w), s) != cudaSuccess) return LMOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return LMOE_ERR_CUDA;
  if (info) *info = w[1];
  return static_cast<lmoe_status>(w[0]);
}

lmoe_status lmoe_route(const lmoe_config* cfg, const void* x, const void* w_router, const float* bias,
                       const float* logits_in, int32_t* topk_idx, float* topk_w, float* logits_out,
                       void* ws, size_t ws_bytes, void* stream) {
  lmoe_status st = check_config(cfg);
  if (st != LMOE_OK) return st;
  if (!topk_idx || !topk_w) return LMOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < layout(cfg, LMOE_OP_ROUTE).total) return LMOE_ERR_WORKSPACE;
  if (!logits_in && (!x || !w_router)) return LMOE_ERR_INVALID_ARG;
  if (!logits_in && cfg->N % 8) return LMOE_ERR_UNSUPPORTED;   // router GEMM: 16-byte logit stores
  if (!aligned16(x) || !aligned16(w_router)) return LMOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Layout L = layout(cfg, LMOE_OP_ROUTE);
  uint32_t* err = err_word(ws);
  const float* logits = logits_in;
  if (!logits) {
    float* lg = logits_out ? logits_out : at<float>(ws, L.logits);
    if (cfg->act == LMOE_F32) {
      SimtLaunch S;
      S.rows = static_cast<int>(cfg->T);
      S.cols = cfg->N;
      S.k = cfg->d;
      S.a = static_cast<const float*>(x);
      S.b = static_cast<const float*>(w_router);
      S.out = lg;
      S.ld_out = cfg->N;
      S.bias = bias;
      S.epi = EPI_F32_BIAS;
      st = simt_gemm(S, err, s);
    } else {
      st = dense_bf16(x, cfg->T, w_router, cfg->N, cfg->d, lg, cfg->N, EPI_F32_BIAS, bias, nullptr, 0,
                      L.splitk ? at<float>(ws, L.splitk) : (L.rsplit ? at<float>(ws, L.rsplit) : nullptr), err, s);
    }
    if (st != LMOE_OK) return st;
    logits = lg;
  }
  // computed logits get their near-tied decisions refined exactly; caller
  // logits are taken as they are
  const bool refine = logits_in == nullptr;
  return launch_topk(logits, cfg->T, cfg->N, cfg->K, topk_idx, topk_w, refine ? x : nullptr,
                     refine ? w_router : nullptr, refine ? bias : nullptr, cfg->d, cfg->act, err, s);
}

lmoe_status lmoe_permute(const lmoe_config* cfg, const int32_t* topk_idx, int32_t* offsets, int32_t* perm_src,
                         int32_t* inv_perm, int32_t* padded_offsets, const void* rows, int64_t row_bytes,
                         void* permuted_rows, const uint8_t* rows_sf, uint8_t* permuted_sf,
                         const float* topk_w, float* perm_gate, void* ws, size_t ws_bytes, void* stream) {
  lmoe_status st = check_config(cfg);
  if (st != LMOE_OK) return st;
  if (!offsets || !padded_offsets) return LMOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!topk_idx || !perm_src || !inv_perm)) return LMOE_ERR_INVALID_ARG;   // T = 0: offsets only
  if ((rows == nullptr) != (permuted_rows == nullptr)) return LMOE_ERR_INVALID_ARG;
  if (rows && (row_bytes <= 0 || row_bytes % 16 || !aligned16(rows) || !aligned16(permuted_rows)))
    return LMOE_ERR_INVALID_ARG;
  if ((rows_sf == nullptr) != (permuted_sf == nullptr)) return LMOE_ERR_INVALID_ARG;
  if (rows_sf && (!rows || (row_bytes * 2) % 64)) return LMOE_ERR_INVALID_ARG;
  if ((topk_w == nullptr) != (perm_gate == nullptr)) return LMOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < layout(cfg, LMOE_OP_PERMUTE).total) return LMOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Layout L = layout(cfg, LMOE_OP_PERMUTE);
  uint32_t* err = err_word(ws);
  st = launch_permute(topk_idx, cfg->T, cfg->K, cfg->N, offsets, perm_src, inv_perm, padded_offsets,
                      at<int32_t>(ws, L.scratch), topk_w, perm_gate, err, s);
  if (st != LMOE_OK) return st;
  if (rows || rows_sf)
    st = launch_gather(topk_idx, perm_src, offsets, padded_offsets, cfg->T * cfg->K, cfg->K, rows, row_bytes,
                       permuted_rows, rows_sf, permuted_sf, cfg->N, s);
  return st;
}

}  // extern "C"

namespace lmoe {
namespace {

// Routed experts on padded expert-grouped rows (BF16 or fp32 experts).
// A dense problem that may ride along in the first expert GEMM's launch:
// out = relu(act . wt^T)^2 (the shared experts' hidden layer).
struct SharedHidden {
  const void* x = nullptr;    // [T][d]
  const void* ws1 = nullptr;  // [S*m_s][d]
  int64_t d = 0;
  int cols = 0;               // S * m_s
  void* out = nullptr;        // [T][S*m_s]
  bool done = false;          // set when it was computed in that launch
  // and their output layer in the second launch: ys = hs . [Ws2_1 .. Ws2_S]^T
  const void* ws2 = nullptr;  // [S][d][m_s]
  int S = 0, ms = 0;
  void* ys = nullptr;         // [T][d]
  bool ys_done = false;
};

lmoe_status expert_ffn_impl(const lmoe_config* cfg, const lmoe_weights* w, const void* zin,
                            const int32_t* offsets, const int32_t* poff, const float* gate, void* a,
                            void* y, uint32_t* err, cudaStream_t s,
                            const std::function<void()>& between = std::function<void()>(),
                            SharedHidden* shared = nullptr) {
  const int64_t P = padded_rows(cfg);
  lmoe_status st;
  if (cfg->act == LMOE_F32) {
    SimtLaunch g1;
    g1.grouped = 1;
    g1.rows = static_cast<int>(P);
    g1.cols = cfg->m;
    g1.k = cfg->l;
    g1.a = static_cast<const float*>(zin);
    g1.b = static_cast<const float*>(w->w1);
    g1.offsets = offsets;
    g1.padded_offsets = poff;
    g1.groups = cfg->N;
    g1.out = static_cast<float*>(a);
    g1.ld_out = cfg->m;
    g1.epi = EPI_SQRELU;
    if ((st = simt_gemm(g1, err, s)) != LMOE_OK) return st;
    if (between) between();
    SimtLaunch g2 = g1;
    g2.cols = cfg->l;
    g2.k = cfg->m;
    g2.a = static_cast<const float*>(a);
    g2.b = static_cast<const float*>(w->w2);
    g2.out = static_cast<float*>(y);
    g2.ld_out = cfg->l;
    g2.epi = EPI_GATE;
    g2.row_scale = gate;
    return simt_gemm(g2, err, s);
  }
  // Weight-major tiles for every grouped GEMM: 128 weight rows x up to BN
  // tokens of one expert, the MMA's N set per tile, so no token padding is
  // multiplied; small token counts use narrow tiles.
  const int sbn = swap_bn(cfg->T) ? swap_bn(cfg->T) : 256;
  const int64_t single_tiles = static_cast<int64_t>(cfg->T) * cfg->K / sbn + cfg->N;
  TcLaunch g1;
  g1.grouped = 1;
  g1.rows = static_cast<int>(P);   // padded rows (bounds of the debug build's checks)
  g1.cols = cfg->m;
  g1.kblocks[0] = kblocks(cfg->l);
  g1.offsets = offsets;
  g1.padded_offsets = poff;
  g1.groups = cfg->N;
  const TcOperand zop{zin, cfg->l, P, 1};
  const TcOperand w1op{w->w1, cfg->l, cfg->m, cfg->N};
  g1.swap = 1;
  g1.bn = sbn;
  g1.a[0] = w1op;
  g1.b[0] = zop;
  g1.max_tiles = single_tiles * ((cfg->m + 127) / 128);
  g1.out = a;
  g1.ld_out = cfg->m;
  g1.epi = EPI_SQRELU;
  // enough tokens per expert on average: CTA pairs, 256 features x 256 tokens per tile
  const bool pairs = sbn == 256 && static_cast<int64_t>(cfg->T) * cfg->K >= 64LL * cfg->N;
  const int64_t pair_token_tiles = static_cast<int64_t>(cfg->T) * cfg->K / 256 + cfg->N;
  if (pairs) {
    g1.max_tiles = pair_token_tiles * ((cfg->m + 255) / 256);
    if (shared && shared->cols > 0) {
      g1.x_act = TcOperand{shared->x, shared->d, cfg->T, 1};
      g1.x_wt = TcOperand{shared->ws1, shared->d, shared->cols, 1};
      g1.rows_x = static_cast<int>(cfg->T);
      g1.cols_x = shared->cols;
      g1.out_x = shared->out;
      g1.ld_out_x = shared->cols;
    }
    st = tc2_gemm(g1, err, s);
    if (st == LMOE_OK && shared && shared->cols > 0) shared->done = true;
  } else {
    st = tc_gemm(g1, err, s);
  }
  if (st != LMOE_OK) return st;
  if (between) between();
  TcLaunch g2 = g1;
  g2.rows_x = 0;   // the extra problem belongs to the first launch only
  g2.cols_x = 0;
  g2.out_x = nullptr;
  g2.cols = cfg->l;
  g2.kblocks[0] = kblocks(cfg->m);
  const TcOperand aop{a, cfg->m, P, 1};
  const TcOperand w2op{w->w2, cfg->m, cfg->l, cfg->N};
  g2.a[0] = w2op;
  g2.b[0] = aop;
  g2.max_tiles = single_tiles * ((cfg->l + 127) / 128);
  g2.out = y;
  g2.ld_out = cfg->l;
  g2.epi = EPI_GATE;
  g2.row_scale = gate;
  if (pairs) {
    g2.max_tiles = pair_token_tiles * ((cfg->l + 255) / 256);
    const bool with_ys = shared && shared->done && shared->ys;
    if (with_ys) {
      g2.x_act = TcOperand{shared->out, static_cast<int64_t>(shared->S) * shared->ms, cfg->T, 1};
      g2.x_wt = TcOperand{shared->ws2, shared->ms, shared->d, shared->S};
      g2.x_kgroup = shared->ms;
      g2.rows_x = static_cast<int>(cfg->T);
      g2.cols_x = static_cast<int>(shared->d);
      g2.out_x = shared->ys;
      g2.ld_out_x = shared->d;
    }
    st = tc2_gemm(g2, err, s);
    if (st == LMOE_OK && with_ys) shared->ys_done = true;
    return st;
  }
  return tc_gemm(g2, err, s);
}

// Routed experts with NVFP4 weights and latent activations: two block-scaled
// GEMMs; the first quantises a = relu(h)^2 to NVFP4 (static scale) in its epilogue.
lmoe_status expert_ffn_fp4(const lmoe_config* cfg, const lmoe_weights* w, const void* zcodes, const uint8_t* zsf,
                           const float* z_gs, const int32_t* offsets, const int32_t* poff, const float* gate,
                           void* a_codes, uint8_t* a_sf, void* y, uint32_t* err, cudaStream_t s,
                           const std::function<void()>& between = std::function<void()>()) {
  const int64_t P = padded_rows(cfg);
  Fp4Launch g1;
  g1.a_codes = zcodes;
  g1.a_sf = zsf;
  g1.a_rows = P;
  g1.b_codes = w->w1;
  g1.b_sf = w->w1_sf;
  g1.k = cfg->l;
  g1.cols = cfg->m;
  g1.groups = cfg->N;
  g1.offsets = offsets;
  g1.padded_offsets = poff;
  g1.in_scale = z_gs;
  g1.w_scale = w->w1_gs;
  g1.out_scale = w->a_global_scale;
  g1.quant_out = 1;
  g1.out = a_codes;
  g1.out_sf = a_sf;
  lmoe_status st = fp4_gemm(g1, err, s);
  if (st != LMOE_OK) return st;
  if (between) between();
  Fp4Launch g2 = g1;
  g2.a_codes = a_codes;
  g2.a_sf = a_sf;
  g2.b_codes = w->w2;
  g2.b_sf = w->w2_sf;
  g2.k = cfg->m;
  g2.cols = cfg->l;
  g2.in_scale = w->a_global_scale;
  g2.w_scale = w->w2_gs;
  g2.out_scale = nullptr;
  g2.row_scale = gate;
  g2.quant_out = 0;
  g2.out = y;
  g2.out_sf = nullptr;
  g2.ld_out = cfg->l;
  return fp4_gemm(g2, err, s);
}

bool fp4_weights_ok(const lmoe_weights* w) {
  return w->w1_sf && w->w2_sf && w->w1_gs && w->w2_gs && w->a_global_scale && aligned16(w->w1_sf) &&
         aligned16(w->w2_sf);
}

}  // namespace
}  // namespace lmoe

extern "C" {

lmoe_status lmoe_expert_ffn(const lmoe_config* cfg, const lmoe_weights* w, const void* permuted_in,
                            const uint8_t* permuted_sf, const float* in_global_scale, const int32_t* offsets,
                            const int32_t* padded_offsets, const float* perm_gate, void* y_perm, void* ws,
                            size_t ws_bytes, void* stream) {
  lmoe_status st = check_config(cfg);
  if (st != LMOE_OK) return st;
  if (!w || !w->w1 || !w->w2 || !permuted_in || !offsets || !padded_offsets || !y_perm)
    return LMOE_ERR_INVALID_ARG;
  if (!aligned16(permuted_in) || !aligned16(y_perm) || !aligned16(w->w1) || !aligned16(w->w2))
    return LMOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < layout(cfg, LMOE_OP_EXPERT_FFN).total) return LMOE_ERR_WORKSPACE;
  const Layout L = layout(cfg, LMOE_OP_EXPERT_FFN);
  if (cfg->expert == LMOE_NVFP4) {
    if (!permuted_sf || !in_global_scale || !fp4_weights_ok(w) || !aligned16(permuted_sf)) return LMOE_ERR_INVALID_ARG;
    return expert_ffn_fp4(cfg, w, permuted_in, permuted_sf, in_global_scale, offsets, padded_offsets, perm_gate,
                          at<void>(ws, L.a), at<uint8_t>(ws, L.a_sf), y_perm, err_word(ws),
                          static_cast<cudaStream_t>(stream));
  }
  return expert_ffn_impl(cfg, w, permuted_in, offsets, padded_offsets, perm_gate, at<void>(ws, L.a), y_perm,
                         err_word(ws), static_cast<cudaStream_t>(stream));
}

lmoe_status lmoe_combine(const lmoe_config* cfg, const void* y_perm, const int32_t* topk_idx,
                         const int32_t* inv_perm, const int32_t* offsets, const int32_t* padded_offsets,
                         const float* topk_w, void* c, void* stream) {
  lmoe_status st = check_config(cfg);
  if (st != LMOE_OK) return st;
  if (!y_perm || !topk_idx || !inv_perm || !offsets || !padded_offsets || !c) return LMOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(c)) return LMOE_ERR_INVALID_ARG;
  return launch_combine(y_perm, cfg->act, topk_idx, inv_perm, offsets, padded_offsets, topk_w, nullptr, c, cfg->T,
                        cfg->K, cfg->N, cfg->l, static_cast<cudaStream_t>(stream));
}

lmoe_status lmoe_nvfp4_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols, const float* global_in,
                                uint8_t* codes, uint8_t* sf, float* global_out, int sf_layout, void* ws,
                                size_t ws_bytes, void* stream) {
  if (!in || !codes || !sf) return LMOE_ERR_INVALID_ARG;
  if (rows < 0 || cols <= 0 || cols % 16) return LMOE_ERR_INVALID_ARG;
  if (in_dtype != LMOE_F32 && in_dtype != LMOE_BF16) return LMOE_ERR_INVALID_ARG;
  const int base_layout = sf_layout & ~LMOE_SF_BLOCK_16X16;
  if (base_layout != LMOE_SF_ROWMAJOR && base_layout != LMOE_SF_MMA_TILED) return LMOE_ERR_INVALID_ARG;
  if (!aligned16(in) || (reinterpret_cast<uintptr_t>(codes) & 7)) return LMOE_ERR_INVALID_ARG;
  lmoe_config q{};
  q.T = rows;
  q.l = static_cast<int32_t>(cols);
  if (!ws || ws_bytes < layout(&q, LMOE_OP_NVFP4_QUANTIZE).total) return LMOE_ERR_WORKSPACE;
  const Layout L = layout(&q, LMOE_OP_NVFP4_QUANTIZE);
  if (rows == 0) return LMOE_OK;
  return launch_nvfp4_quantize(in, in_dtype, rows, cols, global_in, codes, sf, global_out, sf_layout,
                               at<float>(ws, L.partials), nvfp4_partials(rows * cols), err_word(ws),
                               static_cast<cudaStream_t>(stream));
}

lmoe_status lmoe_fp8_quantize(const void* in, int in_dtype, int64_t rows, int64_t cols, const float* scale_in,
                              uint8_t* codes, float* scale_out, void* ws, size_t ws_bytes, void* stream) {
  if (!in || !codes || rows < 0 || cols <= 0 || cols % 16) return LMOE_ERR_INVALID_ARG;
  if (in_dtype != LMOE_BF16 && in_dtype != LMOE_F32) return LMOE_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(codes)) return LMOE_ERR_INVALID_ARG;
  float* partials = nullptr;
  int np = 0;
  if (!scale_in) {
    lmoe_config c = {};
    c.T = rows;
    c.l = static_cast<int32_t>(cols);
    const Layout L = layout(&c, LMOE_OP_FP8_QUANTIZE);
    if (!ws || ws_bytes < L.total) return LMOE_ERR_WORKSPACE;
    partials = at<float>(ws, L.partials);
    np = nvfp4_partials(rows * cols);
  }
  return launch_fp8_quantize(in, in_dtype, rows, cols, scale_in, codes, scale_out, partials, np,
                             static_cast<cudaStream_t>(stream));
}

size_t lmoe_nvfp4_quantize_ex_workspace(int64_t rows, int64_t cols) {
  if (rows < 0 || cols <= 0) return 0;
  return 256 + static_cast<size_t>(nvfp4x_partials(rows * (cols / 16 > 0 ? cols / 16 : 1))) * 8;
}

lmoe_status lmoe_nvfp4_quantize_ex(const void* in, int in_dtype, int64_t rows, int64_t cols, uint32_t flags,
                                   uint32_t rht_signs, uint64_t seed, uint32_t sr_stream, const float* global_in,
                                   uint8_t* codes, uint8_t* sf, float* global_out, int sf_layout, void* ws,
                                   size_t ws_bytes, void* stream) {
  if (!in || !codes || !sf || rows < 0 || cols < 0) return LMOE_ERR_INVALID_ARG;
  if (in_dtype != LMOE_BF16 && in_dtype != LMOE_F32) return LMOE_ERR_INVALID_ARG;
  if (flags & ~(LMOE_QX_TRANSPOSE | LMOE_QX_RHT | LMOE_QX_SR)) return LMOE_ERR_INVALID_ARG;
  const int base = sf_layout & ~LMOE_SF_BLOCK_16X16;
  if ((base != LMOE_SF_ROWMAJOR && base != LMOE_SF_MMA_TILED) || (sf_layout & ~(LMOE_SF_BLOCK_16X16 | 1)))
    return LMOE_ERR_INVALID_ARG;
  if ((sf_layout & LMOE_SF_BLOCK_16X16) && (flags & (LMOE_QX_RHT | LMOE_QX_SR))) return LMOE_ERR_INVALID_ARG;
  const bool tr = (flags & LMOE_QX_TRANSPOSE) != 0;
  const int64_t out_cols = tr ? rows : cols;
  if (out_cols % 16) return LMOE_ERR_INVALID_ARG;
  if (!aligned16(in) || (reinterpret_cast<uintptr_t>(codes) & 7)) return LMOE_ERR_INVALID_ARG;
  if (!global_in && (!ws || ws_bytes < lmoe_nvfp4_quantize_ex_workspace(rows, cols))) return LMOE_ERR_WORKSPACE;
  double* partials = ws ? reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + 256) : nullptr;
  return launch_nvfp4_quantize_ex(in, in_dtype, rows, cols, flags, rht_signs, seed, sr_stream, global_in, codes, sf,
                                  global_out, sf_layout, partials, static_cast<cudaStream_t>(stream));
}

lmoe_status lmoe_nvfp4_transpose_2d(const uint8_t* codes, const uint8_t* sf, int64_t groups, int64_t rows,
                                    int64_t cols, uint8_t* codes_t, uint8_t* sf_t, void* stream) {
  return launch_nvfp4_transpose2d(codes, sf, groups, rows, cols, codes_t, sf_t, static_cast<cudaStream_t>(stream));
}

lmoe_status lmoe_nvfp4_gemm(int groups, const int32_t* offsets, const int32_t* padded_offsets, int64_t a_rows,
                            const uint8_t* a_codes, const uint8_t* a_sf, const float* a_global,
                            int a_global_per_group, const uint8_t* b_codes, const uint8_t* b_sf,
                            const float* b_global, int cols, int64_t k, const float* row_scale, void* out,
                            int64_t ld_out, void* ws, size_t ws_bytes, void* stream) {
  if (groups <= 0 || !offsets || !padded_offsets || !a_codes || !a_sf || !a_global || !b_codes || !b_sf ||
      !b_global || !out)
    return LMOE_ERR_INVALID_ARG;
  if (a_rows < 0 || a_rows % 128 || a_rows > (int64_t(1) << 30) || cols <= 0 || k <= 0 || ld_out < cols)
    return LMOE_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_sf) || !aligned16(b_codes) || !aligned16(b_sf) || !aligned16(out) ||
      (ld_out * 2) % 16)
    return LMOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < 256) return LMOE_ERR_WORKSPACE;
  Fp4Launch g;
  g.a_codes = a_codes;
  g.a_sf = a_sf;
  g.a_rows = a_rows;
  g.b_codes = b_codes;
  g.b_sf = b_sf;
  g.k = k;
  g.cols = cols;
  g.groups = groups;
  g.offsets = offsets;
  g.padded_offsets = padded_offsets;
  g.in_scale = a_global;
  g.in_scale_grouped = a_global_per_group != 0;
  g.w_scale = b_global;
  g.row_scale = row_scale;
  g.quant_out = 0;
  g.out = out;
  g.ld_out = ld_out;
  return fp4_gemm(g, err_word(ws), static_cast<cudaStream_t>(stream));
}

lmoe_status lmoe_forward(const lmoe_config* cfg, const lmoe_weights* w, const void* x, void* out, void* ws,
                         size_t ws_bytes, void* stream) {
  return lmoe_forward_traced(cfg, w, x, out, ws, ws_bytes, stream, nullptr);
}

lmoe_status lmoe_forward_traced(const lmoe_config* cfg, const lmoe_weights* w, const void* x, void* out,
                                void* ws, size_t ws_bytes, void* stream, void* const* events) {
  lmoe_status st = check_config(cfg);
  if (st != LMOE_OK) return st;
  if (!w || !w->w_router || !w->w1 || !w->w2) return LMOE_ERR_INVALID_ARG;
  const bool ident = identity(cfg);
  if (ident != (w->w_down == nullptr) || ident != (w->w_up == nullptr)) return LMOE_ERR_INVALID_ARG;
  if (cfg->n_shared && (!w->ws1 || !w->ws2)) return LMOE_ERR_INVALID_ARG;
  if (shared_fp8(cfg) && (!w->ws1_scale || !w->ws2_scale || !w->shared_x_scale || !w->shared_h_scale))
    return LMOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < layout(cfg, LMOE_OP_FORWARD).total) return LMOE_ERR_WORKSPACE;
  const bool fp4 = cfg->expert == LMOE_NVFP4;
  if (fp4 && !fp4_weights_ok(w)) return LMOE_ERR_INVALID_ARG;
  if (cfg->T == 0) return LMOE_OK;
  if (!x || !out || !aligned16(x) || !aligned16(out)) return LMOE_ERR_INVALID_ARG;
  if (cfg->N % 8) return LMOE_ERR_UNSUPPORTED;   // the router GEMM stores logit rows in 16-byte vectors
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Layout L = layout(cfg, LMOE_OP_FORWARD);
  uint32_t* err = err_word(ws);
  const int64_t T = cfg->T;
  int next_event = 0;
  auto mark = [&](int upto) {
    // record every event up to and including stage `upto` (skipped stages share a time)
    while (events && next_event <= upto) cudaEventRecord(static_cast<cudaEvent_t>(events[next_event++]), s);
  };
  mark(0);
  const int d = cfg->d, l = cfg->l, N = cfg->N, K = cfg->K;
  const size_t ab = act_bytes(cfg);
  const bool f32 = cfg->act == LMOE_F32;
  float* splitk = L.splitk ? at<float>(ws, L.splitk) : nullptr;
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* gw = at<float>(ws, L.w);
  float* logits = at<float>(ws, L.logits);

  // BF16 layer at prefill sizes: the permutation runs first, then (latent
  // projections) the down-projection stores z once, and a token-order copy
  // reads each z row (x with identity projections) once and writes it to the
  // padded rows of its K slots
  const bool scatter_z = !fp4 && !f32 && T > kSwapMaxTokens && l >= 64;
  // The top-K and the permutation need only the router logits, the
  // down-projection only x: when both follow, the routing runs on a side
  // stream beside the down-projection GEMM (whose persistent CTAs leave room
  // on every SM for the routing's small ones). Not while tracing stages.
  SideStream side;
  const bool overlap = !events && !ident && (scatter_z || fp4) && side_stream(&side);
  cudaStream_t rs = overlap ? side.stream : s;

  // 1. router logits (+ bias) and top-K gates
  if (f32) {
    SimtLaunch S;
    S.rows = static_cast<int>(T);
    S.cols = N;
    S.k = d;
    S.a = static_cast<const float*>(x);
    S.b = static_cast<const float*>(w->w_router);
    S.out = logits;
    S.ld_out = N;
    S.bias = w->router_bias;
    S.epi = EPI_F32_BIAS;
    st = simt_gemm(S, err, s);
  } else {
    st = dense_bf16(x, T, w->w_router, N, d, logits, N, EPI_F32_BIAS, w->router_bias, nullptr, 0,
                    L.rsplit ? at<float>(ws, L.rsplit) : splitk, err, s);
  }
  if (st != LMOE_OK) return st;
  if (overlap && (cudaEventRecord(side.fork, s) != cudaSuccess || cudaStreamWaitEvent(rs, side.fork, 0) != cudaSuccess))
    return LMOE_ERR_CUDA;
  if ((st = launch_topk(logits, T, N, K, idx, gw, x, w->w_router, w->router_bias, d, cfg->act, err, rs)) != LMOE_OK)
    return st;
  mark(1);
  // the main stream waits for the routing (no-op without the side stream)
  auto join_routing = [&]() {
    return !overlap || (cudaEventRecord(side.join, rs) == cudaSuccess && cudaStreamWaitEvent(s, side.join, 0) ==
                        cudaSuccess);
  };

  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* poff = at<int32_t>(ws, L.poff);
  int32_t* perm_src = at<int32_t>(ws, L.perm_src);
  int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
  float* gate = at<float>(ws, L.gate);
  void* zp = at<void>(ws, L.zp);
  float* z_gs = nullptr;
  if (scatter_z) {
    int32_t* slot_row = at<int32_t>(ws, L.slot_row);
    if ((st = launch_permute(idx, T, K, N, offsets, perm_src, inv_perm, poff, at<int32_t>(ws, L.scratch), gw, gate,
                             err, rs, kPermSlotsPerWarp, slot_row)) != LMOE_OK)
      return st;
    const void* zb = x;
    if (!ident) {
      void* z = at<void>(ws, L.z);
      if ((st = dense_bf16(x, T, w->w_down, l, d, z, l, EPI_BF16, nullptr, nullptr, 0, splitk, err, s)) != LMOE_OK)
        return st;
      zb = z;
    }
    if (!join_routing()) return LMOE_ERR_CUDA;
    mark(2);
    if ((st = launch_scatter_rows(zb, T, static_cast<int64_t>(l) * ab, slot_row, K, zp, s)) != LMOE_OK) return st;
    mark(3);
  } else if (fp4) {
    // NVFP4 latent activations (current per-tensor amax): the permutation runs
    // first and the quantiser writes each token's codes and scales straight to
    // the padded rows of its K slots
    int32_t* slot_row = at<int32_t>(ws, L.slot_row);
    if ((st = launch_permute(idx, T, K, N, offsets, perm_src, inv_perm, poff, at<int32_t>(ws, L.scratch), gw, gate,
                             err, rs, kPermSlotsPerWarp, slot_row)) != LMOE_OK)
      return st;
    const void* z = x;
    if (!ident) {
      void* zb = at<void>(ws, L.z);
      if ((st = dense_bf16(x, T, w->w_down, l, d, zb, l, EPI_BF16, nullptr, nullptr, 0, splitk, err, s)) != LMOE_OK)
        return st;
      z = zb;
    }
    if (!join_routing()) return LMOE_ERR_CUDA;
    z_gs = at<float>(ws, L.z_gs);
    if ((st = launch_nvfp4_quantize_scatter(z, T, l, slot_row, K, static_cast<uint8_t*>(zp), at<uint8_t>(ws, L.zp_sf),
                                            z_gs, at<float>(ws, L.partials), nvfp4_partials(T * l), s)) != LMOE_OK)
      return st;
    mark(3);
  } else {
    // 2. latent down-projection d -> l
    const void* z = x;
    if (!ident) {
      void* zb = at<void>(ws, L.z);
      if (f32) {
        SimtLaunch S;
        S.rows = static_cast<int>(T);
        S.cols = l;
        S.k = d;
        S.a = static_cast<const float*>(x);
        S.b = static_cast<const float*>(w->w_down);
        S.out = static_cast<float*>(zb);
        S.ld_out = l;
        S.epi = EPI_BF16;
        st = simt_gemm(S, err, s);
      } else {
        st = dense_bf16(x, T, w->w_down, l, d, zb, l, EPI_BF16, nullptr, nullptr, 0, splitk, err, s);
      }
      if (st != LMOE_OK) return st;
      z = zb;
    }
    mark(2);

    // 3. dispatch grouped by expert (padded rows), gates per padded row
    if ((st = launch_permute(idx, T, K, N, offsets, perm_src, inv_perm, poff, at<int32_t>(ws, L.scratch), gw, gate,
                             err, s)) != LMOE_OK)
      return st;
    const int64_t row_bytes = static_cast<int64_t>(l) * ab;
    if ((st = launch_gather(idx, perm_src, offsets, poff, T * K, K, z, row_bytes, zp, nullptr, nullptr, N, s)) !=
        LMOE_OK)
      return st;
    mark(3);
  }

  // 4. routed expert FFNs in l, gate applied in the second GEMM's epilogue; the
  // shared experts' hidden layer (BF16) is offered to the first GEMM's launch
  const int S = cfg->n_shared, ms = cfg->m_shared;
  void* hs = S ? at<void>(ws, L.hs) : nullptr;
  SharedHidden shared_hidden;
  const bool fp8sh = shared_fp8(cfg);
  if (S && !f32 && !fp4 && !fp8sh) {
    shared_hidden.x = x;
    shared_hidden.ws1 = w->ws1;
    shared_hidden.d = d;
    shared_hidden.cols = S * ms;
    shared_hidden.out = hs;
    shared_hidden.ws2 = w->ws2;
    shared_hidden.S = S;
    shared_hidden.ms = ms;
    shared_hidden.ys = at<void>(ws, L.ys);
  }
  void* y = at<void>(ws, L.y);
  const std::function<void()> between = events ? std::function<void()>([&]() { mark(4); }) : std::function<void()>();
  if (fp4)
    st = expert_ffn_fp4(cfg, w, zp, at<uint8_t>(ws, L.zp_sf), z_gs, offsets, poff, gate, at<void>(ws, L.a),
                        at<uint8_t>(ws, L.a_sf), y, err, s, between);
  else
    st = expert_ffn_impl(cfg, w, zp, offsets, poff, gate, at<void>(ws, L.a), y, err, s, between,
                         shared_hidden.cols > 0 ? &shared_hidden : nullptr);
  if (st != LMOE_OK) return st;
  mark(5);

  // 5. combine; with identity projections it is the output when there are no
  // shared experts or their output ys is already there (then combine adds it)
  bool ys_ready = shared_hidden.ys_done;
  // FP8 shared experts: with identity projections their output is added by the
  // combine, so it is computed first; otherwise with the up-projection (stage 7)
  auto run_shared_fp8 = [&]() {
    return shared_experts_fp8(cfg, w, x, at<uint8_t>(ws, L.xq), at<uint8_t>(ws, L.hs), at<void>(ws, L.ys), splitk,
                              err, s);
  };
  if (fp8sh && ident) {
    if ((st = run_shared_fp8()) != LMOE_OK) return st;
    ys_ready = true;
  }
  const bool combine_is_out = ident && (cfg->n_shared == 0 || ys_ready);
  void* c = combine_is_out ? out : at<void>(ws, L.c);
  if ((st = launch_combine(y, cfg->act, idx, inv_perm, offsets, poff, nullptr, ident && ys_ready ? at<void>(ws, L.ys)
                           : nullptr, c, T, K, N, l, s)) != LMOE_OK)
    return st;
  mark(6);
  if (combine_is_out) {
    mark(7);
    return LMOE_OK;
  }

  // 6. shared experts' hidden layer on the d-dim x: hs = relu(x Ws1^T)^2, all S at
  // once (already done when it rode along in the first expert GEMM's launch)
  if (fp8sh && !ys_ready) {
    if ((st = run_shared_fp8()) != LMOE_OK) return st;
    ys_ready = true;
  } else if (S && !shared_hidden.done) {
    if (f32) {
      SimtLaunch G;
      G.rows = static_cast<int>(T);
      G.cols = S * ms;
      G.k = d;
      G.a = static_cast<const float*>(x);
      G.b = static_cast<const float*>(w->ws1);
      G.out = static_cast<float*>(hs);
      G.ld_out = static_cast<int64_t>(S) * ms;
      G.epi = EPI_SQRELU;
      st = simt_gemm(G, err, s);
    } else {
      st = dense_bf16(x, T, w->ws1, S * ms, d, hs, static_cast<int64_t>(S) * ms, EPI_SQRELU, nullptr, nullptr, 0,
                      splitk, err, s);
    }
    if (st != LMOE_OK) return st;
  }

  // 7. up-projection l -> d plus the shared experts' output layer
  if (f32) {
    if (!ident) {
      SimtLaunch U;
      U.rows = static_cast<int>(T);
      U.cols = d;
      U.k = l;
      U.a = static_cast<const float*>(c);
      U.b = static_cast<const float*>(w->w_up);
      U.out = static_cast<float*>(out);
      U.ld_out = d;
      U.epi = EPI_BF16;
      if ((st = simt_gemm(U, err, s)) != LMOE_OK) return st;
    }
    for (int sh = 0; sh < S; ++sh) {
      // out (+)= hs_s Ws2_s^T, hs_s = columns [sh*ms, (sh+1)*ms) of hs
      SimtLaunch U;
      U.rows = static_cast<int>(T);
      U.cols = d;
      U.k = ms;
      U.b = static_cast<const float*>(w->ws2) + static_cast<int64_t>(sh) * d * ms;
      U.out = static_cast<float*>(out);
      U.ld_out = d;
      U.a = static_cast<const float*>(hs) + static_cast<int64_t>(sh) * ms;
      U.lda = static_cast<int64_t>(S) * ms;
      if (ident && sh == 0) {
        U.epi = EPI_ADD_RES;
        U.residual = static_cast<const float*>(c);
        U.ld_res = l;
      } else {
        U.epi = EPI_BF16;
        U.accumulate = 1;
      }
      if ((st = simt_gemm(U, err, s)) != LMOE_OK) return st;
    }
    mark(7);
    return LMOE_OK;
  }

  TcLaunch U;
  U.rows = static_cast<int>(T);
  U.cols = d;
  U.out = out;
  U.ld_out = d;
  U.epi = EPI_BF16;
  const int sbn = swap_bn(T);
  int sg = 0;
  // segment: (activation operand, weight operand, K, weight K-group)
  auto add_seg = [&](TcOperand act, TcOperand wt, int64_t k, int wgroup) {
    if (sbn) {
      U.a[sg] = wt;
      U.b[sg] = act;
      U.a_kgroup[sg] = wgroup;
    } else {
      U.a[sg] = act;
      U.b[sg] = wt;
      U.b_kgroup[sg] = wgroup;
    }
    U.kblocks[sg] = kblocks(k);
    ++sg;
  };
  if (!ident) add_seg(TcOperand{c, l, T, 1}, TcOperand{w->w_up, l, d, 1}, l, 0);
  if (S && !ys_ready)
    add_seg(TcOperand{hs, static_cast<int64_t>(S) * ms, T, 1}, TcOperand{w->ws2, ms, d, S},
            static_cast<int64_t>(S) * ms, ms);
  U.nseg = sg;
  if (ident) {
    U.epi = EPI_ADD_RES;
    U.residual = c;
    U.ld_res = l;
  } else if (ys_ready) {   // out = c W_up^T + ys
    U.epi = EPI_ADD_RES;
    U.residual = at<void>(ws, L.ys);
    U.ld_res = d;
  }
  if (sbn) {
    U.swap = 1;
    U.bn = sbn;
    U.max_tiles = (d + 127) / 128;
    U.ksplit = choose_splits(U.max_tiles, U.kblocks[0] + (U.nseg > 1 ? U.kblocks[1] : 0), splitk);
    U.partial = splitk;
  } else {
    U.bn = normal_bn(d);
    U.max_tiles = ((T + 127) / 128) * ((d + U.bn - 1) / U.bn);
  }
  st = tc_gemm(U, err, s);
  mark(7);
  return st;
}

}  // extern "C"
