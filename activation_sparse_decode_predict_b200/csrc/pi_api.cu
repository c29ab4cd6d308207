// pi_api.cu -- the C ABI of libpi (declared in include/pi.h): argument checks,
// workspace layout and launch sequences.  Nothing here allocates device memory.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "pi.h"
#include "pi_args.h"
#include "pi_attn.cuh"
#include "pi_batch.cuh"
#include "pi_common.cuh"
#include "pi_kernels_v1.cuh"
#include "pi_layout.h"
#include "pi_stack.cuh"
#include "pi_tc.cuh"

namespace {

thread_local char g_err[512] = "no error";

pi_status fail(pi_status st, const char* fmt, const char* what) {
  snprintf(g_err, sizeof(g_err), fmt, what);
  return st;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// the token-block FFN kernels (pi_set_token_block_ffn); process-wide
std::atomic<int> g_token_ffn{PI_TOKEN_FFN_WARP_MMA};

// whether a token block of this shape takes the tcgen05 FFN
bool use_tc_ffn(int wtype, int ttype, int d, int B) {
  return g_token_ffn.load(std::memory_order_relaxed) == PI_TOKEN_FFN_TCGEN05 && pi::tc_ffn_supported(wtype, ttype, d, B);
}

}  // namespace

namespace pi {

void set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

pi_status check_desc(const pi_ffn_desc* d, int32_t batch) {
  if (!d) return fail(PI_ERR_INVALID_ARG, "%s", "desc is NULL");
  if (d->d <= 0 || d->d % 8) return fail(PI_ERR_INVALID_ARG, "%s", "d must be a positive multiple of 8");
  if (d->ffn <= 0) return fail(PI_ERR_INVALID_ARG, "%s", "ffn must be positive");
  if (d->n_hot < 0 || d->n_hot > d->ffn) return fail(PI_ERR_INVALID_ARG, "%s", "n_hot must be in [0, ffn]");
  if (d->rank <= 0 || d->rank % 8) return fail(PI_ERR_INVALID_ARG, "%s", "rank must be a positive multiple of 8");
  if (d->wtype != PI_F32 && d->wtype != PI_F16 && d->wtype != PI_Q4_0)
    return fail(PI_ERR_INVALID_ARG, "%s", "wtype must be PI_F32, PI_F16 or PI_Q4_0");
  if (d->ptype != PI_F32 && d->ptype != PI_F16 && d->ptype != PI_Q4_0)
    return fail(PI_ERR_INVALID_ARG, "%s", "ptype must be PI_F32, PI_F16 or PI_Q4_0");
  if (d->ptype == PI_Q4_0 && (d->d % 32 || d->rank % 32))
    return fail(PI_ERR_INVALID_ARG, "%s", "a Q4_0 predictor needs d % 32 == 0 and rank % 32 == 0");
  if (d->act != PI_ACT_RELU && d->act != PI_ACT_REGLU && d->act != PI_ACT_RELU2)
    return fail(PI_ERR_INVALID_ARG, "%s", "act must be PI_ACT_RELU, PI_ACT_REGLU or PI_ACT_RELU2");
  if (d->wtype == PI_Q4_0 && d->d % 32) return fail(PI_ERR_INVALID_ARG, "%s", "Q4_0 needs d % 32 == 0");
  if (batch < 1 || batch > PI_MAX_BATCH) return fail(PI_ERR_INVALID_ARG, "%s", "batch must be in [1, 16]");
  if (d->d > 16384) return fail(PI_ERR_UNSUPPORTED, "%s", "d above 16384 is not supported");
  if (d->rank > 65536) return fail(PI_ERR_UNSUPPORTED, "%s", "rank above 65536 is not supported");
  return PI_OK;
}

pi_status check_ptr(const void* p, size_t align, const char* name) {
  if (!p) return fail(PI_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, align)) return fail(PI_ERR_INVALID_ARG, "%s is not aligned", name);
  return PI_OK;
}

}  // namespace pi

namespace {

using pi::check_desc;
using pi::check_ptr;

#ifdef PI_TRACE
// profiling builds: where the decode-step kernel writes its phase stamps
uint64_t* g_trace = nullptr;
#endif

pi_status cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_err, sizeof(g_err), "%s: %s", where, cudaGetErrorString(e));
  return PI_ERR_CUDA;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

pi_status check_weight(const pi_ffn_desc* d, pi_weight w, const char* name) {
  pi_status s = check_ptr(w.data, 16, name);
  if (s) return s;
  if (d->wtype == PI_Q4_0) {
    s = check_ptr(w.scales, 16, "Q4_0 scales");
    if (s) return s;
  }
  return PI_OK;
}

pi_status check_ws(const pi_ffn_desc* d, int32_t batch, void* ws, size_t ws_bytes) {
  pi_status s = check_ptr(ws, 256, "ws");
  if (s) return s;
  if (ws_bytes < pi_workspace_bytes(d, batch))
    return fail(PI_ERR_CAPACITY, "%s", "workspace smaller than pi_workspace_bytes()");
  return PI_OK;
}

#define PI_TRY(x)                   \
  do {                              \
    pi_status _s = (x);             \
    if (_s != PI_OK) return _s;     \
  } while (0)
#define PI_CUDA(x, where)                          \
  do {                                             \
    cudaError_t _e = (x);                          \
    if (_e != cudaSuccess) return cuda_fail(_e, where); \
  } while (0)

pi_status predict_impl(const pi_ffn_desc* d, int32_t B, const void* h, const void* P1, const void* P2,
                       const float* bp, float thr, int32_t* idx, int32_t* count, char* ws, cudaStream_t st) {
  const pi::WsLayout L = pi::ws_layout(d->d, d->ffn, d->n_hot, d->rank, B);
  float* u = reinterpret_cast<float*>(ws + L.u);
  uint32_t* tmask = reinterpret_cast<uint32_t*>(ws + L.tile_mask);
  int* tcount = reinterpret_cast<int*>(ws + L.tile_count);
  const int C = d->ffn - d->n_hot;
  const int sms = sm_count();
  if (pi::batch_pred_supported(d->ptype, d->d, d->rank, B)) {
    // token blocks of 3..16 with fp16 predictors: tensor-core P1 and P2 (scratch:
    // P1 dots in the partials, scores in the pre-activations)
    PI_CUDA(pi::launch_batch_predict(h, B, d->d, d->rank, C, d->n_hot, P1, P2, bp, thr,
                                     reinterpret_cast<float*>(ws + L.partial),
                                     reinterpret_cast<float*>(ws + L.pre), tmask, tcount,
                                     reinterpret_cast<pi::Ctrl*>(ws), sms, st),
            "tensor-core predictor launch");
    PI_CUDA(pi::launch_compact(tmask, tcount, C, d->n_hot, idx, count, st), "compaction launch");
    return PI_OK;
  }
  PI_CUDA(pi::launch_pred_u(d->ptype, P1, pi::pred_scales(d, P1, d->rank, d->d), h, B, d->d, d->rank, u, sms, st),
          "predictor GEMV1 launch");
  PI_CUDA(pi::launch_pred_score(d->ptype, P2, pi::pred_scales(d, P2, C, d->rank), bp, u, B, d->rank, C, thr, tmask,
                                tcount, st),
          "predictor score launch");
  PI_CUDA(pi::launch_compact(tmask, tcount, C, d->n_hot, idx, count, st), "compaction launch");
  return PI_OK;
}

pi_status ffn_impl(const pi_ffn_desc* d, int32_t B, const void* h, const int32_t* idx, const int32_t* count,
                   pi_weight Wg, pi_weight Wu, pi_weight Wd, const float* b1, const float* b2, float* y, char* ws,
                   cudaStream_t st) {
  const pi::WsLayout L = pi::ws_layout(d->d, d->ffn, d->n_hot, d->rank, B);
  int* status = reinterpret_cast<int*>(ws);
  float* a = reinterpret_cast<float*>(ws + L.act);
  float* partial = reinterpret_cast<float*>(ws + L.partial);
  const int sms = sm_count();
  const int ht = pi::token_type(d);
  if (use_tc_ffn(d->wtype, ht, d->d, B)) {
    // token blocks of 3..16 with fp16 weights: gathered tiles on tcgen05, fp32
    // accumulators in tensor memory, y (with b2) written by the last kernel
    PI_CUDA(pi::launch_tc_ffn(d->act, h, B, d->d, d->ffn, d->n_hot, idx, count, Wg.data, Wu.data, Wd.data, b1, b2, y,
                              ws + L.tc, reinterpret_cast<pi::Ctrl*>(ws), sms, st),
            "tcgen05 FFN launch");
    return PI_OK;
  }
  if (pi::batch_supported(d->wtype, ht, d->d, B)) {
    // token blocks of 3..16: tensor-core gate/up, down on the tensor cores
    // (fp16 weights) or on the CUDA cores (Q4_0)
    const int NR = d->wtype == PI_Q4_0 ? pi::down_ranges(d->d, sms) : pi::batch_ranges(d->d, sms);
    PI_CUDA(pi::launch_batch_ffn(d->act, d->wtype, h, B, d->d, d->ffn, d->n_hot, idx, count, Wg.data, Wg.scales,
                                 Wu.data, Wu.scales, Wd.data, Wd.scales, b1, reinterpret_cast<float*>(ws + L.pre),
                                 partial, NR, reinterpret_cast<pi::Ctrl*>(ws), sms, st),
            "tensor-core FFN launch");
    PI_CUDA(pi::launch_ffn_reduce(partial, NR, B, d->d, b2, y, st), "split-K reduce launch");
    return PI_OK;
  }
  const int G = pi::down_ranges(d->d, sms);
  PI_CUDA(pi::launch_ffn_act(d->wtype, ht, d->act, h, B, d->d, d->ffn, d->n_hot, idx, count, Wg.data,
                             Wg.scales, Wu.data, Wu.scales, b1, a, d->ffn, status, sms, st),
          "FFN activation launch");
  PI_CUDA(pi::launch_ffn_down(d->wtype, B, d->d, d->ffn, d->n_hot, idx, count, Wd.data, Wd.scales, a, d->ffn,
                              partial, G, st),
          "FFN down launch");
  PI_CUDA(pi::launch_ffn_reduce(partial, G, B, d->d, b2, y, st), "split-K reduce launch");
  return PI_OK;
}

pi_status check_layer(const pi_ffn_desc* desc, const pi_layer_weights* w) {
  PI_TRY(check_ptr(w->P1, 16, "P1"));
  if (desc->ffn > desc->n_hot) PI_TRY(check_ptr(w->P2, 16, "P2"));
  if (w->bp) PI_TRY(check_ptr(w->bp, 4, "bp"));
  if (desc->act == PI_ACT_REGLU) PI_TRY(check_weight(desc, w->W_gate, "W_gate"));
  PI_TRY(check_weight(desc, w->W_up, "W_up"));
  PI_TRY(check_weight(desc, w->W_downT, "W_downT"));
  if (w->b1) PI_TRY(check_ptr(w->b1, 4, "b1"));
  if (w->b2) PI_TRY(check_ptr(w->b2, 16, "b2"));
  if (w->rank != 0) {
    const int unit = desc->ptype == PI_Q4_0 ? 32 : 8;
    if (w->rank < 0 || w->rank % unit || w->rank > desc->rank)
      return fail(PI_ERR_INVALID_ARG, "%s",
                  "a layer's rank must be 0 (the descriptor's) or a multiple of 8 (Q4_0 predictors: 32) "
                  "no larger than the descriptor's rank");
  }
  return PI_OK;
}

// The descriptor of one layer: the layer's own predictor rank when it has one.
pi_ffn_desc layer_desc(const pi_ffn_desc* desc, const pi_layer_weights* w) {
  pi_ffn_desc d = *desc;
  if (w->rank > 0) d.rank = w->rank;
  return d;
}

pi_status check_attn(const pi_attn_desc* d, int32_t batch) {
  if (!d) return fail(PI_ERR_INVALID_ARG, "%s", "desc is NULL");
  if (d->d <= 0 || d->d % 8) return fail(PI_ERR_INVALID_ARG, "%s", "d must be a positive multiple of 8");
  if (d->n_heads <= 0 || d->d % d->n_heads) return fail(PI_ERR_INVALID_ARG, "%s", "n_heads must divide d");
  if (!pi::attn_head_dim_ok(d->d / d->n_heads))
    return fail(PI_ERR_UNSUPPORTED, "%s", "head dimension must be 32, 64, 128 or 256");
  if (d->n_hot < 0 || d->n_hot > d->n_heads) return fail(PI_ERR_INVALID_ARG, "%s", "n_hot must be in [0, n_heads]");
  if (d->s_max <= 0) return fail(PI_ERR_INVALID_ARG, "%s", "s_max must be positive");
  if (d->wtype != PI_F16 && d->wtype != PI_F32) return fail(PI_ERR_INVALID_ARG, "%s", "wtype must be PI_F16 or PI_F32");
  if (d->xtype != PI_F16 && d->xtype != PI_F32) return fail(PI_ERR_INVALID_ARG, "%s", "xtype must be PI_F16 or PI_F32");
  if (d->ctype != PI_F16 && d->ctype != PI_F32) return fail(PI_ERR_INVALID_ARG, "%s", "ctype must be PI_F16 or PI_F32");
  if (d->wtype == PI_F16 && d->xtype == PI_F32)
    return fail(PI_ERR_UNSUPPORTED, "%s", "fp32 tokens need fp32 weights");
  if (batch < 1 || batch > PI_MAX_BATCH) return fail(PI_ERR_INVALID_ARG, "%s", "batch must be in [1, 16]");
  return PI_OK;
}

// Workspace of pi_sparse_attention: [ctrl][q, k, v of the listed heads][chunk
// partials][head outputs][W_o^T row list][its count][split-K partial outputs]
struct AttnLayout {
  size_t qkv, part, a, orow, ocount, partial, total;
};

AttnLayout attn_layout(const pi_attn_desc* d, int32_t B) {
  AttnLayout L;
  const size_t dh = (size_t)(d->d / d->n_heads);
  size_t off = pi::kCtrlBytes;
  L.qkv = off; off += pi::align256((size_t)B * d->n_heads * 3 * dh * 4);
  L.part = off; off += pi::align256((size_t)B * d->n_heads * pi::kAttnMaxSplit * (dh + 4) * 4);
  L.a = off; off += pi::align256((size_t)B * d->d * 4);
  L.orow = off; off += pi::align256((size_t)d->d * 4);
  L.ocount = off; off += 256;
  L.partial = off; off += pi::align256((size_t)pi::kGMax * B * d->d * 4);
  L.total = off;
  return L;
}

// The head predictor as pi_predict sees it: the heads are its neurons.
pi_ffn_desc head_desc(const pi_ffn_desc* f, const pi_attn_desc* a, int32_t head_rank) {
  pi_ffn_desc h = *f;
  h.ffn = a->n_heads;
  h.n_hot = a->n_hot;
  h.rank = head_rank;
  return h;
}

// Workspace of pi_decode_blocks: [FFN workspace][head predictor workspace]
// [attention workspace][attention output B x d fp32][g, h: B x d tokens each]
struct BlocksLayout {
  size_t ffn, head, attn, ya, g, h, total, ffn_bytes, attn_bytes;
};

pi_status blocks_layout(const pi_ffn_desc* f, const pi_attn_desc* a, int32_t B, BlocksLayout& L) {
  PI_TRY(check_desc(f, B));
  PI_TRY(check_attn(a, B));
  if (a->d != f->d) return fail(PI_ERR_INVALID_ARG, "%s", "the attention and FFN descriptors must share d");
  if (a->xtype != pi::token_type(f)) return fail(PI_ERR_INVALID_ARG, "%s", "adesc->xtype must be the token type");
  const pi_ffn_desc hd = head_desc(f, a, f->rank);
  PI_TRY(check_desc(&hd, B));
  size_t off = 0;
  L.ffn = off;
  L.ffn_bytes = pi_workspace_bytes(f, B);
  off += pi::align256(L.ffn_bytes);
  L.head = off;
  off += pi::align256(pi_workspace_bytes(&hd, B));
  L.attn = off;
  L.attn_bytes = attn_layout(a, B).total;
  off += pi::align256(L.attn_bytes);
  const size_t tok = (size_t)B * f->d * (pi::token_type(f) == PI_F32 ? 4 : 2);
  L.ya = off; off += pi::align256((size_t)B * f->d * 4);
  L.g = off; off += pi::align256(tok);
  L.h = off; off += pi::align256(tok);
  L.total = off;
  return PI_OK;
}

static_assert(pi::kYAccCopies == pi::kYCopies, "workspace layout and kernel agree on the accumulator copies");
static_assert(pi::kGMax == pi::kGMaxCtas, "workspace layout and kernel agree on the largest grid");
static_assert(pi::kLayersMax == pi::kMaxLayers && pi::kLayersMax == PI_MAX_LAYERS, "layer limits agree");
static_assert(sizeof(pi::Ctrl) == pi::kCtrlBytes, "control block size");
static_assert(sizeof(pi::Ctrl{}.pool) / sizeof(int) == pi::kLayersMax, "one claim counter per layer");

int stack_grid() {
  const int g = sm_count();
  return g < pi::kGMax ? g : pi::kGMax;
}

// Fill the persistent kernel's parameters; PI_ERR_UNSUPPORTED if the shape
// does not fit its constraints (the caller then runs the per-kernel path).
pi_status fused_params(const pi_ffn_desc* desc, int32_t B, int32_t n_layers, pi::StackParams& P, size_t& smem,
                       int& G) {
  if (!pi::stack_supported(desc->wtype, desc->ptype, desc->d, desc->ffn, desc->n_hot, desc->rank, B, n_layers))
    return PI_ERR_UNSUPPORTED;
  G = stack_grid();
  memset(&P, 0, sizeof(P));
  P.d = desc->d;
  P.ffn = desc->ffn;
  P.n_hot = desc->n_hot;
  P.rank = desc->rank;
  P.act = desc->act;
  P.L = n_layers;
  P.T = desc->d / pi::stack_ept(desc->d);
  smem = pi::stack_smem_layout(P, desc->ptype, B, G);
  if (smem == 0) return PI_ERR_UNSUPPORTED;
  const int ep = desc->ptype == PI_F16 ? 2 : 4;
  const size_t wrow = desc->wtype == PI_Q4_0 ? desc->d / 2 + desc->d / 16
                                              : (size_t)desc->d * (desc->wtype == PI_F16 ? 2 : 4);
  const size_t neuron = (wrow + 16) * (desc->act == PI_ACT_REGLU ? 3 : 2) + 16 + 256;
  // predictor items (the largest rank): fp16 predictors go to the tensor cores
  // in 16-row tiles with padded rows; Q4_0 rows carry codes and scales
  const size_t p2item = desc->ptype == PI_F16    ? (size_t)16 * (2 * desc->rank + 16) + 256
                        : desc->ptype == PI_Q4_0 ? (size_t)(P.T / 32) * (desc->rank / 2 + desc->rank / 16) + 256
                                                 : (size_t)(P.T / 32) * desc->rank * ep;
  const size_t p1item = desc->ptype == PI_Q4_0 ? (size_t)desc->d / 2 + desc->d / 16 + 256 : (size_t)desc->d * ep + 256;
  const size_t half = (size_t)P.ring_bytes / 2;
  if (neuron > half || p2item > half || p1item > half) return PI_ERR_UNSUPPORTED;
  // the tensor-core P1 tile takes at most 16 rows, and the rows of one tile
  // (each a ring item of 2d bytes plus alignment and skew) fill at most half the ring
  P.p1rows = 16;
  if (desc->ptype == PI_F16) {
    const int fit = (int)(half / ((size_t)desc->d * 2 + 240));
    if (fit < P.p1rows) P.p1rows = fit;
    if (P.p1rows < 1) return PI_ERR_UNSUPPORTED;
  }
  // a group of ng neurons stays resident while the next group streams in:
  // ng items fill at most half the ring; a tensor-core group's gate and up
  // rows fill one 16-row tile
  const int rpn = desc->act == PI_ACT_REGLU ? 2 : 1;
  {
    // a consumer holds one group while it waits for the first item of the next
    // one, and a wrap of the ring can waste up to one item: ng + 2 items fit
    const int cap = pi::kNgFull ? (int)((size_t)P.ring_bytes / neuron) - 2 : (int)(half / neuron);
    // CUDA-core groups: 4 neurons; Q4_0 rows with a Q4_0 predictor or a token
    // block of 2: 6 (13B-shaped stack: +2.8 % and +4.7 %; with an fp16
    // predictor and one token 6 lost 3 % and 8 lost 3-6 % everywhere)
    const int lim = (desc->wtype == PI_F16 && desc->ptype == PI_F16 && pi::kF16Mma) ? 16 / rpn
                    : (desc->wtype == PI_Q4_0 && (desc->ptype == PI_Q4_0 || B == 2)) ? 6
                                                                                         : 4;
    P.ng = cap < lim ? cap : lim;
    if (P.ng < 1) P.ng = 1;
  }
  // a few groups of hot neurons per CTA are shared out statically (they fill
  // the wait for barrier U and the list's latency after P2); the rest is
  // claimed, which balances the CTAs
  {
    // wide rows (d >= 8192) leave only 2-3 neurons per group, and barrier U
    // takes longer there: three groups fill its wait, six with gated rows
    // (measured: 70B-shaped ReGLU 12 neurons per CTA against 6: +0.7-0.9 % at
    // sparsity 0.80-0.95, 24 -2 %; 40B-shaped ReLU: 9 best, 12 -0.6 %, 3 -3.4 %)
    const int def_a = desc->d >= 8192 ? (rpn == 2 ? 6 : 3) * P.ng : P.ng;
    // the share after P2: one group, two on wide gated rows (70B-shaped: +0.4 %;
    // 7B / 13B-shaped: a larger share after P2 changed nothing or lost 2.5 %)
    const int def_b = desc->d >= 8192 && rpn == 2 ? 2 * P.ng : P.ng;
    const int per_a = pi::kHotA > 0 ? pi::kHotA : def_a, per_b = pi::kHotB > 0 ? pi::kHotB : def_b;
    P.hot_a = desc->n_hot < G * per_a ? desc->n_hot : G * per_a;
    P.hot_static = desc->n_hot - P.hot_a < G * per_b ? desc->n_hot : P.hot_a + G * per_b;
    // with fewer claimed hot neurons than one group per CTA the claims cannot
    // even out the CTAs' predicted cold rows, so every row above a CTA's
    // running mean is handed over; with a larger pool a slack of two rows
    // saves the hand-over round trips (measured: 7B / 13B +2 %, 40B / 70B -1 %
    // and -0.4 % with no slack); one row on gated rows (70B-shaped: +0.35 %
    // over two, -1.7 % with four; 40B-shaped ReLU keeps two: one lost 0.6 %)
    P.don_slack = desc->n_hot - P.hot_static < G * P.ng ? 0 : (rpn == 2 ? 1 : 2);
  }
  const int C = desc->ffn - desc->n_hot;
  // every consumer thread holds at most kShareRegs entries of the CTA's P2 bias share
  if ((C + G - 1) / G > pi::kShareRegs * P.T) return PI_ERR_UNSUPPORTED;
  // the final list compaction keeps cmp_layers layers of this CTA's list (and
  // two offsets per layer) in the ring
  P.cmp_layers = (int)((size_t)P.ring_bytes / ((size_t)P.seg_cap * 4 + 8));
  if (P.cmp_layers < 1) return PI_ERR_UNSUPPORTED;
  return PI_OK;
}

pi_status fused_stack(const pi_ffn_desc* desc, int32_t B, int32_t n_layers, const pi_layer_weights* layers,
                      const void* h_in, void* h_out, int32_t* idx, int32_t* counts, float* y, void* h_trace, float eps,
                      char* ws, const pi::WsLayout& L, cudaStream_t st) {
  pi::StackParams P;
  size_t smem = 0;
  int G = 0;
  const pi_status fs = fused_params(desc, B, n_layers, P, smem, G);
  if (fs != PI_OK) return fs;
  P.eps = eps;
  P.h_in = h_in;
  P.h_out = h_out;
  P.idx = idx;
  P.counts = counts;
  P.y_out = y;
  P.h_trace = h_trace;
  P.ctrl = reinterpret_cast<pi::Ctrl*>(ws);
  P.u_g = reinterpret_cast<float*>(ws + L.u);
  P.yacc = reinterpret_cast<float*>(ws + L.yacc);
  P.pool = reinterpret_cast<pi::Ctrl*>(ws)->pool;
  P.lcnt = reinterpret_cast<int*>(ws + L.lcnt);
  P.don = reinterpret_cast<int*>(ws + L.don);
#ifdef PI_TRACE
  P.trace = g_trace;
#endif
  for (int l = 0; l < n_layers; ++l) {
    const pi_layer_weights& w = layers[l];
    pi::StackLayer& s = P.layers[l];
    s.P1 = w.P1;
    s.P2 = w.P2;
    s.bp = w.bp;
    s.wg = w.W_gate.data;
    s.wg_sc = w.W_gate.scales;
    s.wu = w.W_up.data;
    s.wu_sc = w.W_up.scales;
    s.wd = w.W_downT.data;
    s.wd_sc = w.W_downT.scales;
    s.b1 = w.b1;
    s.b2 = w.b2;
    // a neuron item carries the 16-byte block of b1 that holds its bias
    if (w.b1 && (reinterpret_cast<uintptr_t>(w.b1) & 15u)) return PI_ERR_UNSUPPORTED;
    s.thr = w.threshold;
    s.rank = w.rank > 0 ? w.rank : desc->rank;
    if (!pi::stack_rank_ok(desc->ptype, s.rank)) return PI_ERR_UNSUPPORTED;
    const pi_ffn_desc ld = layer_desc(desc, &w);
    s.P1_sc = pi::pred_scales(&ld, w.P1, s.rank, desc->d);
    s.P2_sc = pi::pred_scales(&ld, w.P2, desc->ffn - desc->n_hot, s.rank);
  }
  PI_CUDA(pi::launch_stack(desc->wtype, desc->ptype, B, P, G, smem, st), "fused decode-step launch");
  return PI_OK;
}

}  // namespace

extern "C" {

#ifdef PI_TRACE
// profiling builds only: [n_layers, grid, kTraceEvents] uint64 device buffer (or NULL)
PI_API void pi_trace_buffer(void* buf) { g_trace = static_cast<uint64_t*>(buf); }
#endif

const char* pi_last_error(void) { return g_err; }

const char* pi_version(void) { return "0.1.0"; }

size_t pi_workspace_bytes(const pi_ffn_desc* desc, int32_t batch) {
  if (check_desc(desc, batch) != PI_OK) return 0;
  return pi::ws_layout(desc->d, desc->ffn, desc->n_hot, desc->rank, batch).total;
}

pi_status pi_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  PI_TRY(check_ptr(ws, 256, "ws"));
  if (ws_bytes < sizeof(pi::Ctrl)) return fail(PI_ERR_CAPACITY, "%s", "workspace smaller than its control block");
  // the whole workspace: the control block and the hand-over slots of the
  // persistent kernel must start at zero (the kernel leaves them zero)
  PI_CUDA(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream), "workspace init");
  return PI_OK;
}

pi_status pi_predict(const pi_ffn_desc* desc, int32_t batch, const void* h, const void* P1, const void* P2,
                     const float* bp, float threshold, int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                     void* stream) {
  PI_TRY(check_desc(desc, batch));
  PI_TRY(check_ptr(h, 16, "h"));
  PI_TRY(check_ptr(P1, 16, "P1"));
  if (desc->ffn > desc->n_hot) PI_TRY(check_ptr(P2, 16, "P2"));
  if (bp) PI_TRY(check_ptr(bp, 4, "bp"));
  if (desc->ffn > desc->n_hot) PI_TRY(check_ptr(idx, 4, "idx"));
  PI_TRY(check_ptr(count, 4, "count"));
  PI_TRY(check_ws(desc, batch, ws, ws_bytes));
  return predict_impl(desc, batch, h, P1, P2, bp, threshold, idx, count, (char*)ws, (cudaStream_t)stream);
}

pi_status pi_sparse_ffn(const pi_ffn_desc* desc, int32_t batch, const void* h, const int32_t* idx,
                        const int32_t* count, pi_weight W_gate, pi_weight W_up, pi_weight W_downT, const float* b1,
                        const float* b2, float* y, void* ws, size_t ws_bytes, void* stream) {
  PI_TRY(check_desc(desc, batch));
  PI_TRY(check_ptr(h, 16, "h"));
  if (desc->ffn > desc->n_hot) PI_TRY(check_ptr(idx, 4, "idx"));
  PI_TRY(check_ptr(count, 4, "count"));
  if (desc->act == PI_ACT_REGLU) PI_TRY(check_weight(desc, W_gate, "W_gate"));
  PI_TRY(check_weight(desc, W_up, "W_up"));
  PI_TRY(check_weight(desc, W_downT, "W_downT"));
  if (b1) PI_TRY(check_ptr(b1, 4, "b1"));
  if (b2) PI_TRY(check_ptr(b2, 16, "b2"));
  PI_TRY(check_ptr(y, 16, "y"));
  PI_TRY(check_ws(desc, batch, ws, ws_bytes));
  return ffn_impl(desc, batch, h, idx, count, W_gate, W_up, W_downT, b1, b2, y, (char*)ws, (cudaStream_t)stream);
}

pi_status pi_layer(const pi_ffn_desc* desc, int32_t batch, const void* h, const pi_layer_weights* w, int32_t* idx,
                   int32_t* count, float* y, void* ws, size_t ws_bytes, void* stream) {
  if (!w) return fail(PI_ERR_INVALID_ARG, "%s", "layer weights are NULL");
  PI_TRY(check_desc(desc, batch));
  PI_TRY(check_ptr(h, 16, "h"));
  PI_TRY(check_ptr(w->P1, 16, "P1"));
  if (desc->ffn > desc->n_hot) PI_TRY(check_ptr(w->P2, 16, "P2"));
  if (w->bp) PI_TRY(check_ptr(w->bp, 4, "bp"));
  if (desc->ffn > desc->n_hot) PI_TRY(check_ptr(idx, 4, "idx"));
  PI_TRY(check_ptr(count, 4, "count"));
  if (desc->act == PI_ACT_REGLU) PI_TRY(check_weight(desc, w->W_gate, "W_gate"));
  PI_TRY(check_weight(desc, w->W_up, "W_up"));
  PI_TRY(check_weight(desc, w->W_downT, "W_downT"));
  if (w->b1) PI_TRY(check_ptr(w->b1, 4, "b1"));
  if (w->b2) PI_TRY(check_ptr(w->b2, 16, "b2"));
  PI_TRY(check_ptr(y, 16, "y"));
  PI_TRY(check_ws(desc, batch, ws, ws_bytes));
  PI_TRY(check_layer(desc, w));
  cudaStream_t st = (cudaStream_t)stream;
  const pi_ffn_desc ld = layer_desc(desc, w);
  PI_TRY(predict_impl(&ld, batch, h, w->P1, w->P2, w->bp, w->threshold, idx, count, (char*)ws, st));
  return ffn_impl(desc, batch, h, idx, count, w->W_gate, w->W_up, w->W_downT, w->b1, w->b2, y, (char*)ws, st);
}

pi_status pi_residual_rmsnorm(int32_t batch, int32_t d, pi_dtype htype, const void* h, const float* y, float eps,
                              void* h_out, void* stream) {
  if (batch < 1 || batch > PI_MAX_BATCH) return fail(PI_ERR_INVALID_ARG, "%s", "batch must be in [1, 16]");
  if (d <= 0 || d % 8) return fail(PI_ERR_INVALID_ARG, "%s", "d must be a positive multiple of 8");
  if (htype != PI_F32 && htype != PI_F16) return fail(PI_ERR_INVALID_ARG, "%s", "htype must be PI_F32 or PI_F16");
  if (!(eps >= 0.f)) return fail(PI_ERR_INVALID_ARG, "%s", "eps must be >= 0");
  if (d > 16384) return fail(PI_ERR_UNSUPPORTED, "%s", "d above 16384 is not supported");
  PI_TRY(check_ptr(h, 16, "h"));
  PI_TRY(check_ptr(y, 16, "y"));
  PI_TRY(check_ptr(h_out, 16, "h_out"));
  PI_CUDA(pi::launch_rmsnorm(htype, h, y, batch, d, eps, h_out, (cudaStream_t)stream), "rmsnorm launch");
  return PI_OK;
}

pi_status pi_decode_stack(const pi_ffn_desc* desc, int32_t batch, int32_t n_layers, const pi_layer_weights* layers,
                          const void* h_in, void* h_out, int32_t* idx, int32_t* counts, float* y, void* h_trace,
                          float eps, void* ws, size_t ws_bytes, void* stream) {
  PI_TRY(check_desc(desc, batch));
  if (n_layers < 1 || n_layers > PI_MAX_LAYERS) return fail(PI_ERR_INVALID_ARG, "%s", "n_layers must be in [1, 128]");
  if (h_trace) PI_TRY(check_ptr(h_trace, 16, "h_trace"));
  if (!layers) return fail(PI_ERR_INVALID_ARG, "%s", "layers is NULL");
  PI_TRY(check_ptr(h_in, 16, "h_in"));
  PI_TRY(check_ptr(h_out, 16, "h_out"));
  if (h_in == h_out) return fail(PI_ERR_INVALID_ARG, "%s", "h_out must not alias h_in");
  if (desc->ffn > desc->n_hot) PI_TRY(check_ptr(idx, 4, "idx"));
  PI_TRY(check_ptr(counts, 4, "counts"));
  if (y) PI_TRY(check_ptr(y, 16, "y"));
  if (!(eps >= 0.f)) return fail(PI_ERR_INVALID_ARG, "%s", "eps must be >= 0");
  PI_TRY(check_ws(desc, batch, ws, ws_bytes));
  for (int l = 0; l < n_layers; ++l) PI_TRY(check_layer(desc, &layers[l]));
  const pi::WsLayout L = pi::ws_layout(desc->d, desc->ffn, desc->n_hot, desc->rank, batch);
  char* wsc = (char*)ws;
  {
    const pi_status fs = fused_stack(desc, batch, n_layers, layers, h_in, h_out, idx, counts, y, h_trace, eps, wsc, L,
                                     (cudaStream_t)stream);
    if (fs != PI_ERR_UNSUPPORTED) return fs;
  }
  float* ybuf = reinterpret_cast<float*>(wsc + L.ybuf);
  void* hbuf[2] = {h_out, wsc + L.hbuf};
  const size_t C = (size_t)(desc->ffn - desc->n_hot);
  cudaStream_t st = (cudaStream_t)stream;
  // h_l ping-pongs between a workspace buffer and h_out so that the last layer lands in h_out.
  const void* cur = h_in;
  const size_t hbytes = (size_t)batch * desc->d * (desc->ptype == PI_F32 ? 4 : 2);
  for (int l = 0; l < n_layers; ++l) {
    if (h_trace) PI_CUDA(cudaMemcpyAsync((char*)h_trace + l * hbytes, cur, hbytes, cudaMemcpyDeviceToDevice, st),
                         "h trace copy");
    float* yl = y ? y + (size_t)l * batch * desc->d : ybuf;
    PI_TRY(pi_layer(desc, batch, cur, &layers[l], idx + (size_t)l * C, counts + l, yl, ws, ws_bytes, stream));
    void* nxt = hbuf[(n_layers - 1 - l) & 1];
    PI_CUDA(pi::launch_rmsnorm(pi::token_type(desc), cur, yl, batch, desc->d, eps, nxt, st), "rmsnorm launch");
    cur = nxt;
  }
  return PI_OK;
}

size_t pi_attn_workspace_bytes(const pi_attn_desc* desc, int32_t batch) {
  if (check_attn(desc, batch) != PI_OK) return 0;
  return attn_layout(desc, batch).total;
}

pi_status pi_sparse_attention(const pi_attn_desc* desc, int32_t batch, const void* x, const int32_t* head_idx,
                              const int32_t* head_count, const void* Wq, const void* Wk, const void* Wv,
                              const void* WoT, void* K, void* V, int32_t len, float* y, void* ws, size_t ws_bytes,
                              void* stream) {
  PI_TRY(check_attn(desc, batch));
  if (len < 0 || len >= desc->s_max) return fail(PI_ERR_INVALID_ARG, "%s", "len must be in [0, s_max)");
  PI_TRY(check_ptr(x, 16, "x"));
  if (desc->n_heads > desc->n_hot) PI_TRY(check_ptr(head_idx, 4, "head_idx"));
  PI_TRY(check_ptr(head_count, 4, "head_count"));
  PI_TRY(check_ptr(Wq, 16, "Wq"));
  PI_TRY(check_ptr(Wk, 16, "Wk"));
  PI_TRY(check_ptr(Wv, 16, "Wv"));
  PI_TRY(check_ptr(WoT, 16, "WoT"));
  PI_TRY(check_ptr(K, 16, "K"));
  PI_TRY(check_ptr(V, 16, "V"));
  PI_TRY(check_ptr(y, 16, "y"));
  PI_TRY(check_ptr(ws, 256, "ws"));
  const AttnLayout L = attn_layout(desc, batch);
  if (ws_bytes < L.total) return fail(PI_ERR_CAPACITY, "%s", "workspace smaller than pi_attn_workspace_bytes()");
  char* w = static_cast<char*>(ws);
  const int sms = sm_count();
  pi::AttnParams P;
  P.d = desc->d;
  P.n_heads = desc->n_heads;
  P.n_hot = desc->n_hot;
  P.B = batch;
  P.s_max = desc->s_max;
  P.len = len;
  P.nsplit = pi::attn_splits(len, batch, desc->n_heads, sms);
  P.x = x;
  P.head_idx = head_idx;
  P.head_count = head_count;
  P.Wq = Wq;
  P.Wk = Wk;
  P.Wv = Wv;
  P.WoT = WoT;
  P.K = K;
  P.V = V;
  P.qkv = reinterpret_cast<float*>(w + L.qkv);
  P.part = reinterpret_cast<float*>(w + L.part);
  P.ctrl = reinterpret_cast<pi::Ctrl*>(w);
  const int G = pi::down_ranges(desc->d, sms);
  PI_CUDA(pi::launch_attention(P, desc->wtype, desc->xtype, desc->ctype, reinterpret_cast<float*>(w + L.a),
                               reinterpret_cast<int32_t*>(w + L.orow), reinterpret_cast<int32_t*>(w + L.ocount),
                               reinterpret_cast<float*>(w + L.partial), G, y, sms, (cudaStream_t)stream),
          "sparse attention launch");
  return PI_OK;
}

size_t pi_blocks_workspace_bytes(const pi_ffn_desc* fdesc, const pi_attn_desc* adesc, int32_t batch) {
  BlocksLayout L;
  if (blocks_layout(fdesc, adesc, batch, L) != PI_OK) return 0;
  return L.total;
}

pi_status pi_decode_blocks(const pi_ffn_desc* fdesc, const pi_attn_desc* adesc, int32_t batch, int32_t n_layers,
                           const pi_block_weights* layers, const void* h_in, void* h_out, int32_t len,
                           int32_t* head_idx, int32_t* head_counts, int32_t* idx, int32_t* counts, void* trace,
                           float eps, void* ws, size_t ws_bytes, void* stream) {
  BlocksLayout L;
  PI_TRY(blocks_layout(fdesc, adesc, batch, L));
  if (n_layers < 1 || n_layers > PI_MAX_LAYERS) return fail(PI_ERR_INVALID_ARG, "%s", "n_layers must be in [1, 128]");
  if (!layers) return fail(PI_ERR_INVALID_ARG, "%s", "layers is NULL");
  if (len < 0 || len >= adesc->s_max) return fail(PI_ERR_INVALID_ARG, "%s", "len must be in [0, s_max)");
  PI_TRY(check_ptr(h_in, 16, "h_in"));
  PI_TRY(check_ptr(h_out, 16, "h_out"));
  if (h_in == h_out) return fail(PI_ERR_INVALID_ARG, "%s", "h_out must not alias h_in");
  PI_TRY(check_ptr(head_idx, 4, "head_idx"));
  PI_TRY(check_ptr(head_counts, 4, "head_counts"));
  if (fdesc->ffn > fdesc->n_hot) PI_TRY(check_ptr(idx, 4, "idx"));
  PI_TRY(check_ptr(counts, 4, "counts"));
  if (trace) PI_TRY(check_ptr(trace, 16, "trace"));
  if (!(eps >= 0.f)) return fail(PI_ERR_INVALID_ARG, "%s", "eps must be >= 0");
  PI_TRY(check_ptr(ws, 256, "ws"));
  if (ws_bytes < L.total) return fail(PI_ERR_CAPACITY, "%s", "workspace smaller than pi_blocks_workspace_bytes()");
  for (int l = 0; l < n_layers; ++l) {
    const pi_block_weights& w = layers[l];
    PI_TRY(check_layer(fdesc, &w.ffn));
    const pi_ffn_desc hd = head_desc(fdesc, adesc, w.head_rank);
    PI_TRY(check_desc(&hd, batch));
    if (w.head_rank > fdesc->rank) return fail(PI_ERR_INVALID_ARG, "%s", "head_rank above the FFN descriptor's rank");
    PI_TRY(check_ptr(w.P1h, 16, "P1h"));
    if (adesc->n_heads > adesc->n_hot) PI_TRY(check_ptr(w.P2h, 16, "P2h"));
    if (w.bph) PI_TRY(check_ptr(w.bph, 4, "bph"));
  }
  char* wsc = static_cast<char*>(ws);
  char* ws_ffn = wsc + L.ffn;
  char* ws_head = wsc + L.head;
  char* ws_attn = wsc + L.attn;
  float* ya = reinterpret_cast<float*>(wsc + L.ya);
  void* gbuf = wsc + L.g;
  void* hbuf[2] = {h_out, wsc + L.h};
  cudaStream_t st = (cudaStream_t)stream;
  const int ht = pi::token_type(fdesc);
  const size_t hbytes = (size_t)batch * fdesc->d * (ht == PI_F32 ? 4 : 2);
  const size_t C = (size_t)(fdesc->ffn - fdesc->n_hot);
  const void* cur = h_in;
  for (int l = 0; l < n_layers; ++l) {
    const pi_block_weights& w = layers[l];
    if (trace)
      PI_CUDA(cudaMemcpyAsync((char*)trace + (size_t)(2 * l) * hbytes, cur, hbytes, cudaMemcpyDeviceToDevice, st),
              "trace copy");
    const pi_ffn_desc hd = head_desc(fdesc, adesc, w.head_rank);
    int32_t* hidx = head_idx + (size_t)l * adesc->n_heads;
    PI_TRY(predict_impl(&hd, batch, cur, w.P1h, w.P2h, w.bph, w.thr_h, hidx, head_counts + l, ws_head, st));
    PI_TRY(pi_sparse_attention(adesc, batch, cur, hidx, head_counts + l, w.Wq, w.Wk, w.Wv, w.WoT, w.K, w.V, len, ya,
                               ws_attn, L.attn_bytes, stream));
    PI_CUDA(pi::launch_rmsnorm(ht, cur, ya, batch, fdesc->d, eps, gbuf, st), "rmsnorm launch");
    if (trace)
      PI_CUDA(cudaMemcpyAsync((char*)trace + (size_t)(2 * l + 1) * hbytes, gbuf, hbytes, cudaMemcpyDeviceToDevice, st),
              "trace copy");
    void* nxt = hbuf[(n_layers - 1 - l) & 1];
    PI_TRY(pi_decode_stack(fdesc, batch, 1, &w.ffn, gbuf, nxt, idx ? idx + (size_t)l * C : nullptr, counts + l,
                           nullptr, nullptr, eps, ws_ffn, L.ffn_bytes, stream));
    cur = nxt;
  }
  return PI_OK;
}

pi_status pi_set_token_block_ffn(int32_t path) {
  if (path != PI_TOKEN_FFN_WARP_MMA && path != PI_TOKEN_FFN_TCGEN05)
    return fail(PI_ERR_INVALID_ARG, "%s", "path must be PI_TOKEN_FFN_WARP_MMA or PI_TOKEN_FFN_TCGEN05");
  g_token_ffn.store(path, std::memory_order_relaxed);
  return PI_OK;
}

int32_t pi_get_token_block_ffn(void) { return g_token_ffn.load(std::memory_order_relaxed); }

int32_t pi_stack_launches(const pi_ffn_desc* desc, int32_t batch, int32_t n_layers) {
  if (check_desc(desc, batch) != PI_OK || n_layers < 1 || n_layers > PI_MAX_LAYERS) return -1;
  {
    pi::StackParams P;
    size_t smem = 0;
    int G = 0;
    if (fused_params(desc, batch, n_layers, P, smem, G) == PI_OK) return 1;
  }
  // the per-layer path: the kernels predict_impl, ffn_impl and the glue launch
  // (memsets are not kernels)
  const bool cold = desc->ffn > desc->n_hot;
  int pred;
  if (pi::batch_pred_supported(desc->ptype, desc->d, desc->rank, batch))
    pred = cold ? 4 : 1;  // P1 and P2 row dots, threshold, compaction
  else
    pred = cold ? 3 : 1;  // u, scores, compaction
  int ffn;
  if (use_tc_ffn(desc->wtype, pi::token_type(desc), desc->d, batch))
    ffn = 2;  // up (+ bias and activation), down (+ the sum over writers and b2)
  else
    ffn = 3;  // gate/up (or row dots), down, reduce
  return (pred + ffn + 1) * n_layers;
}

pi_status pi_get_device_status(void* ws, int32_t* status_out, int32_t clear, void* stream) {
  PI_TRY(check_ptr(ws, 256, "ws"));
  if (!status_out) return fail(PI_ERR_INVALID_ARG, "%s", "status_out is NULL");
  cudaStream_t st = (cudaStream_t)stream;
  int32_t v = 0;
  PI_CUDA(cudaMemcpyAsync(&v, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, st), "status read");
  PI_CUDA(cudaStreamSynchronize(st), "status read sync");
  if (clear) {
    PI_CUDA(cudaMemsetAsync(ws, 0, sizeof(int32_t), st), "status clear");
    PI_CUDA(cudaStreamSynchronize(st), "status clear sync");
  }
  *status_out = v;
  return PI_OK;
}

}  // extern "C"
