/*
 * pi.h -- C ABI of libpi: the activation-sparse decode FFN on one NVIDIA B200.
 *
 * The operation is the per-layer hot path of predictor-driven activation
 * sparsity as the PowerInfer pages describe it:
 *
 *   [GN] GeekNews, "Serving model bahasa besar berkecepatan tinggi pada PC
 *        dengan GPU konsumen"
 *   [AB] aibars.net, "PowerInfer - Hochgeschwindigkeits-Inferenz-Engine für
 *        große Sprachmodelle"
 *   [UA] unite.ai, "PowerInfer: Tüketici Düzeyinde bir GPU ile Hızlı Büyük
 *        Dil Modeli Sunucusu"
 *
 * A small per-layer predictor picks the FFN neurons that will fire ([UA]
 * "Adaptif Sparsite Predictor’ları"); neuron-aware operators then read and
 * compute only those rows of W_gate / W_up and columns of W_down ([UA] "Nöron
 * Bilinçli Operatör"); the always-hot neurons, stored first by the offline
 * layout ([UA] "Nöron Yerleştirme ve Yönetimi"; [AB] "Hot-Cold-Neuron-
 * Mechanismus"), are always computed as one dense slice.
 *
 * Conventions for every entry point
 * ---------------------------------
 * - Every tensor pointer is a DEVICE pointer, owned by the caller, 16-byte
 *   aligned, with dense row-major strides.  The library allocates nothing and
 *   keeps no global state; all scratch lives in the caller's workspace `ws`.
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *   stream).  Calls are asynchronous and ordered on that stream.
 * - Errors the host can see (bad descriptor, NULL or misaligned pointer,
 *   workspace too small, unsupported shape) are returned synchronously and
 *   nothing is launched.  A launch failure returns PI_ERR_CUDA.  Errors found
 *   on the device (an index outside [n_hot, ffn), a count above capacity, a
 *   bounded wait that ran out) set a sticky word in `ws`; read it with
 *   pi_get_device_status().  The kernels never trap.
 * - Calls are reentrant when they use different workspaces.  Calls that share
 *   a workspace must be ordered (same stream, or synchronised).
 * - Storage order is hot-first: neuron rows [0, n_hot) are the hot neurons,
 *   rows [n_hot, ffn) the cold ones.  The neuron table that maps storage rows
 *   back to the model's original rows stays with the caller.
 *
 * Layouts (d = hidden size, F = ffn, H = n_hot, C = F - H, r = rank, B = batch)
 *   h        [B, d]   token block: fp32 when ptype is F32, else fp16
 *   P1       [r, d]   predictor first matrix, `ptype`
 *   P2       [C, r]   predictor second matrix (cold neurons only), `ptype`
 *   A Q4_0 predictor matrix [rows, cols] is ONE buffer: the codes
 *   qs [rows, cols/2] then, right after them, the scales sc [rows, cols/32]
 *   fp16 (32-element blocks along d for P1 and along the rank for P2; the
 *   same block format as the Q4_0 weights below).
 *   bp       [C]      fp32 predictor bias, may be NULL
 *   W_gate   [F, d]   gate rows (ReGLU only), `wtype`
 *   W_up     [F, d]   up rows, `wtype`
 *   W_downT  [F, d]   W_down stored neuron-major (row j = column j of W_down)
 *   b1       [F]      fp32 bias of the gate (ReGLU) or of the up projection,
 *                     may be NULL
 *   b2       [d]      fp32 output bias, may be NULL
 *   y        [B, d]   fp32 output
 *   idx      [C]      int32 active-neuron list, ascending storage rows in
 *                     [H, F); its length lives in the device scalar `count`;
 *                     may be NULL when C == 0
 *   Q4_0 weights use split planes: data = qs [F, d/2] uint8, scales =
 *   sc [F, d/32] fp16; in each 32-element block, byte k holds element k in
 *   its low nibble and element k + 16 in its high nibble, x = s * (q - 8)
 *   ([GN] "Kuantisasi dan kompatibilitas": INT4 Q4_0).
 */
#ifndef PI_H_
#define PI_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PI_API __attribute__((visibility("default")))
#else
#define PI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PI_OK = 0,
  PI_ERR_INVALID_ARG = -1,  /* bad descriptor, NULL/misaligned pointer, bad size */
  PI_ERR_UNSUPPORTED = -2,  /* valid but not implemented (shape/dtype combination) */
  PI_ERR_CUDA = -3,         /* a CUDA call failed; see pi_last_error() */
  PI_ERR_CAPACITY = -4,     /* workspace too small, or a device count above capacity */
  PI_ERR_TIMEOUT = -5,      /* a bounded device-side wait ran out */
  PI_ERR_INDEX = -6         /* device found an active index outside [n_hot, ffn) */
} pi_status;

typedef enum { PI_F32 = 0, PI_F16 = 1, PI_Q4_0 = 2 } pi_dtype;

/* [GN] "Keterbatasan dan FAQ": the supported activation families. */
typedef enum {
  PI_ACT_RELU = 0,   /* a = max(W_up h + b1, 0)                      */
  PI_ACT_REGLU = 1,  /* a = max(W_gate h + b1, 0) * (W_up h)          */
  PI_ACT_RELU2 = 2   /* a = max(W_up h + b1, 0)^2  (not gated)         */
} pi_act;

/* Shape and types of one FFN layer. */
typedef struct {
  int32_t d;       /* hidden size; multiple of 8 (Q4_0: of 32)            */
  int32_t ffn;     /* neurons per layer                                   */
  int32_t n_hot;   /* hot neurons, rows [0, n_hot); 0 <= n_hot <= ffn     */
  int32_t rank;    /* predictor rank (the largest of a stack's layers);
                      multiple of 8 (Q4_0 predictors: of 32)               */
  pi_dtype wtype;  /* FFN weights: PI_F32, PI_F16 or PI_Q4_0             */
  pi_dtype ptype;  /* predictor matrices: PI_F32 (fp32 token block), PI_F16
                      or PI_Q4_0 (fp16 token block); PI_Q4_0 needs d % 32 == 0
                      ([UA] "Adaptif Sparsite Predictor’ları": the predictor's
                      size is chosen per layer; a Q4_0 one is the smallest) */
  pi_act act;
} pi_ffn_desc;

/* One weight matrix: `data` (fp32/fp16 rows, or Q4_0 qs), `scales` (Q4_0 sc, else NULL). */
typedef struct {
  const void *data;
  const void *scales;
} pi_weight;

/* All per-layer tensors of one layer (device pointers). */
typedef struct {
  const void *P1;
  const void *P2;
  const float *bp;
  pi_weight W_gate;   /* ignored unless act == PI_ACT_REGLU */
  pi_weight W_up;
  pi_weight W_downT;
  const float *b1;
  const float *b2;
  float threshold;    /* predictor threshold: neuron c is active iff its score > threshold */
  int32_t rank;       /* this layer's predictor rank, P1 [rank, d] and P2 [C, rank]; 0 = the
                         descriptor's; else a multiple of 8 (Q4_0: 32) no larger than it
                         ([UA] "Adaptif Sparsite Predictor’ları": each layer's predictor has its
                         own size) */
} pi_layer_weights;

/* Maximum token-block size accepted by every call. */
#define PI_MAX_BATCH 16
/* Maximum number of layers of one pi_decode_stack call. */
#define PI_MAX_LAYERS 128

/*
 * Bytes of device workspace a call with this descriptor and batch needs
 * (the largest over pi_predict, pi_sparse_ffn, pi_layer and pi_decode_stack).
 * Returns 0 for an invalid descriptor.  The workspace must be zeroed once
 * (pi_workspace_init) before its first use; the library keeps it consistent
 * afterwards.
 */
PI_API size_t pi_workspace_bytes(const pi_ffn_desc *desc, int32_t batch);

/* Zero the workspace (ws_bytes from ws; status word, counters and the slots
 * the decode-step kernel expects to start at zero), on `stream`. */
PI_API pi_status pi_workspace_init(void *ws, size_t ws_bytes, void *stream);

/*
 * pi_predict -- which cold neurons will fire ([UA] "Adaptif Sparsite
 * Predictor’ları": a per-layer predictor; only predicted-active neurons are
 * computed; [UA] "Çevrim İçi Aşama": the engine predicts active neurons and
 * skips the rest).  The pages do not state the predictor's form; this call
 * computes the low-rank reading
 *     u[b,k] = max(0, sum_i P1[k,i] h[b,i])          (fp32 accumulation)
 *     s[b,c] = sum_k P2[c,k] u[b,k] + bp[c]
 *     active(c) = OR over b of (s[b,c] > threshold)
 * and writes idx = ascending { n_hot + c : active(c) } and *count = |idx|.
 * Hot neurons are not scored: they are always computed.
 *   h [B, d] ptype; P1 [r, d]; P2 [C, r]; bp [C] or NULL;
 *   idx: device int32 [C] (capacity C); count: device int32 scalar.
 * The list is identical to an exact evaluation except for neurons whose
 * score is within rounding (well under 1e-3) of the threshold.
 */
PI_API pi_status pi_predict(const pi_ffn_desc *desc, int32_t batch, const void *h, const void *P1, const void *P2,
                     const float *bp, float threshold, int32_t *idx, int32_t *count, void *ws, size_t ws_bytes,
                     void *stream);

/*
 * pi_sparse_ffn -- the neuron-aware sparse FFN over the list
 * [0, n_hot) ++ idx[0, *count) ([UA] "Nöron Bilinçli Operatör": single rows
 * of the up/gate matrices and single columns of the down matrix, no dense
 * conversion at run time; [GN] "Metode inferensi hibrida CPU/GPU": the dense
 * always-active block runs on the GPU):
 *     for each listed neuron j and token b:
 *         ReGLU:  a = max(W_gate[j].h_b + b1[j], 0) * (W_up[j].h_b)
 *         ReLU:   a = max(W_up[j].h_b + b1[j], 0)
 *         ReLU^2: a = max(W_up[j].h_b + b1[j], 0)^2
 *     y[b, :] = b2 + sum over listed j of a * W_downT[j, :]
 * Every token of the block uses the same list (the union mask).  Dots and the
 * output accumulate in fp32; the activation is kept in fp32, except that
 * token blocks of 3-16 with fp16 weights feed it to the tensor cores as an
 * fp16 pair hi + lo (hi = round(a), lo = round(a - hi), about 22 bits).
 * `count` is read on the device (no host synchronisation); an index outside
 * [n_hot, ffn) or a count above C sets PI_ERR_INDEX / PI_ERR_CAPACITY in the
 * status word and is skipped.
 */
PI_API pi_status pi_sparse_ffn(const pi_ffn_desc *desc, int32_t batch, const void *h, const int32_t *idx,
                        const int32_t *count, pi_weight W_gate, pi_weight W_up, pi_weight W_downT, const float *b1,
                        const float *b2, float *y, void *ws, size_t ws_bytes, void *stream);

/*
 * pi_layer -- pi_predict followed by pi_sparse_ffn on the same token block
 * (one decode step of one FFN layer).  Writes idx/count and y exactly as the
 * two calls would.
 */
PI_API pi_status pi_layer(const pi_ffn_desc *desc, int32_t batch, const void *h, const pi_layer_weights *w, int32_t *idx,
                   int32_t *count, float *y, void *ws, size_t ws_bytes, void *stream);

/*
 * pi_residual_rmsnorm -- glue between stacked FFN layers (the pages do not
 * say what joins the layers; this is the plainest reading that keeps the
 * token statistics fixed): x = h + y;  h_out = x / sqrt(mean(x^2) + eps),
 * computed in fp32 and stored in `htype` (F32 or F16).  h_out may alias h.
 * d <= 16384 (larger: PI_ERR_UNSUPPORTED).
 */
PI_API pi_status pi_residual_rmsnorm(int32_t batch, int32_t d, pi_dtype htype, const void *h, const float *y, float eps,
                              void *h_out, void *stream);

/*
 * pi_decode_stack -- one decode step through `n_layers` layers:
 *     h_0 = h_in;  for l: (idx_l, count_l, y_l) = pi_layer(h_l);
 *                         h_{l+1} = pi_residual_rmsnorm(h_l, y_l, eps)
 *     h_out = h_{n_layers}
 * layers: HOST array of n_layers pi_layer_weights (read during the call; its
 * device pointers are baked into the launch, so a captured CUDA graph keeps
 * them).  idx: [n_layers, C] int32; counts: [n_layers] int32; y: optional
 * [n_layers, B, d] fp32 (NULL: not kept); h_trace: optional [n_layers, B, d]
 * in the token type, receiving each layer's input h_l (NULL: not kept).
 * h_in and h_out [B, d] are in the token type; h_out must not alias h_in.  All layers share one descriptor, except that
 * each layer may have its own (smaller) predictor rank (layers[l].rank);
 * n_layers <= PI_MAX_LAYERS.
 * Token blocks of 1-2 run the whole step as one cooperative launch (one CTA
 * per SM) for fp16/fp16, Q4_0/fp16, Q4_0/Q4_0 and fp32/fp32 weights and
 * predictors, when every b1 is 16-byte aligned and every layer's rank is a
 * multiple of 16 (fp16 predictors) or 256 (Q4_0 predictors); larger blocks
 * and other shapes run per-layer kernels.  Either way the outputs are
 * complete once the stream reaches the end of the call; one workspace
 * serves one call at a time.
 */
PI_API pi_status pi_decode_stack(const pi_ffn_desc *desc, int32_t batch, int32_t n_layers,
                                 const pi_layer_weights *layers, const void *h_in, void *h_out, int32_t *idx,
                                 int32_t *counts, float *y, void *h_trace, float eps, void *ws, size_t ws_bytes,
                                 void *stream);

/*
 * Number of kernel launches one pi_decode_stack call with these arguments
 * issues (for accounting; -1 for invalid arguments).
 */
PI_API int32_t pi_stack_launches(const pi_ffn_desc *desc, int32_t batch, int32_t n_layers);

/*
 * Which kernels run the sparse FFN of a token block of 3-16 tokens with fp16
 * weights and fp16 tokens (d % 256 == 0, d / 256 <= 148):
 *   PI_TOKEN_FFN_WARP_MMA  row-dot kernels on warp-level mma.sync, whole
 *                          contiguous rows per copy (the default: the faster
 *                          of the two on B200 at the 40B/70B shapes)
 *   PI_TOKEN_FFN_TCGEN05   128-neuron tiles gathered by TMA into shared memory,
 *                          tcgen05.mma with fp32 accumulators in tensor memory
 * Both add every sum in a fixed order, so each is deterministic; they differ
 * in rounding order only.  The choice is process-wide and holds for calls
 * issued after it returns (pi_sparse_ffn, pi_layer, pi_decode_stack,
 * pi_decode_blocks and pi_stack_launches).  PI_ERR_INVALID_ARG for any other
 * value.
 */
#define PI_TOKEN_FFN_WARP_MMA 0
#define PI_TOKEN_FFN_TCGEN05 1
PI_API pi_status pi_set_token_block_ffn(int32_t path);
PI_API int32_t pi_get_token_block_ffn(void);

/*
 * Read (and optionally clear) the sticky device status word of `ws`.  Waits
 * for `stream`.  *status_out = PI_OK or the first device-side error recorded.
 */
PI_API pi_status pi_get_device_status(void *ws, int32_t *status_out, int32_t clear, void *stream);

/*
 * Head-sparse decode self-attention ([UA] "Adaptif Sparsite Predictor’ları":
 * besides the FFN predictor, each layer has a predictor for its
 * self-attention block that picks the heads to compute; the other heads are
 * skipped).  The head predictor is pi_predict itself, with the heads as its
 * neurons: a pi_ffn_desc {d, ffn = n_heads, n_hot, rank, ..., ptype} (wtype
 * and act are not used by pi_predict) gives head_idx / head_count.
 */
typedef struct {
  int32_t d;        /* hidden size, multiple of 8                                 */
  int32_t n_heads;  /* heads; head dimension dh = d / n_heads: 32, 64, 128 or 256 */
  int32_t n_hot;    /* always-computed heads [0, n_hot); 0 <= n_hot <= n_heads    */
  int32_t s_max;    /* cache positions per (sequence, head)                      */
  pi_dtype wtype;   /* Wq, Wk, Wv, WoT: PI_F16 or PI_F32                           */
  pi_dtype xtype;   /* token block: PI_F16, or PI_F32 with fp32 weights            */
  pi_dtype ctype;   /* KV cache: PI_F16 or PI_F32                                  */
} pi_attn_desc;

/* Workspace bytes of pi_sparse_attention for this descriptor and batch (0: invalid). */
PI_API size_t pi_attn_workspace_bytes(const pi_attn_desc *desc, int32_t batch);

/*
 * pi_sparse_attention -- one decode step of the self-attention block over the
 * heads [0, n_hot) ++ head_idx[0, *head_count), for a token block of `batch`
 * independent sequences, each with its own cache of `len` positions:
 *     for every listed head h and token b (rows h*dh .. h*dh+dh-1 of each matrix):
 *         q = Wq[h] x_b,  k = Wk[h] x_b,  v = Wv[h] x_b          (fp32)
 *         p = softmax over t = 0..len of q.K[b,h,t] / sqrt(dh), with
 *             K[b,h,len] = k (this step's own k and v are used as computed)
 *         o = sum_t p_t V[b,h,t]
 *         y_b += sum_i o_i WoT[h*dh + i, :]
 *     and k, v are stored (rounded to ctype) at K[b,h,len], V[b,h,len].
 * Unlisted heads are not computed and their cache rows are not written.
 *   x [B, d] xtype; Wq, Wk, Wv [d, d] wtype (head-major rows); WoT [d, d]
 *   wtype = W_o transposed (row h*dh + i is column h*dh + i of W_o);
 *   K, V [B, n_heads, s_max, dh] ctype; 0 <= len < s_max (host value);
 *   head_idx [n_heads - n_hot] int32 (may be NULL when n_hot == n_heads);
 *   head_count: device int32 scalar; y [B, d] fp32 (overwritten).
 * A listed head outside [n_hot, n_heads) sets PI_ERR_INDEX in the workspace
 * status word and is skipped; a count above n_heads - n_hot sets
 * PI_ERR_CAPACITY and is clamped.
 */
PI_API pi_status pi_sparse_attention(const pi_attn_desc *desc, int32_t batch, const void *x,
                                     const int32_t *head_idx, const int32_t *head_count, const void *Wq,
                                     const void *Wk, const void *Wv, const void *WoT, void *K, void *V,
                                     int32_t len, float *y, void *ws, size_t ws_bytes, void *stream);

/*
 * A whole decode step through transformer blocks: per layer the head-sparse
 * self-attention and the activation-sparse FFN, each followed by the stack
 * glue ([UA] "Çevrim İçi Aşama": the engine predicts the active neurons of
 * each layer and computes only those; [UA] "Adaptif Sparsite Predictor’ları":
 * one predictor for the attention heads and one for the FFN neurons).
 */
typedef struct {
  pi_layer_weights ffn;            /* the FFN layer, as for pi_decode_stack                  */
  const void *P1h;                 /* head predictor [head_rank, d], the FFN descriptor's ptype */
  const void *P2h;                 /* [n_heads - n_hot, head_rank] (NULL when every head is hot) */
  const float *bph;                /* [n_heads - n_hot] fp32 or NULL                          */
  const void *Wq, *Wk, *Wv, *WoT;  /* [d, d] each, the attention descriptor's wtype          */
  void *K, *V;                     /* this layer's caches [B, n_heads, s_max, dh]            */
  float thr_h;                     /* head predictor threshold                                */
  int32_t head_rank;               /* head predictor rank: a multiple of 8 (Q4_0: 32), at most
                                      the FFN descriptor's rank                                */
} pi_block_weights;

/* Workspace bytes of pi_decode_blocks (0: invalid descriptors). */
PI_API size_t pi_blocks_workspace_bytes(const pi_ffn_desc *fdesc, const pi_attn_desc *adesc, int32_t batch);

/*
 * pi_decode_blocks -- one decode step of a token block through n_layers blocks:
 *     for l:  heads_l = pi_predict over the heads of h_l (head predictor of layer l)
 *             a_l = pi_sparse_attention(h_l, heads_l, caches of layer l at position len)
 *             g_l = RMSNorm(h_l + a_l)
 *             (idx_l, y_l) = the FFN layer on g_l;  h_{l+1} = RMSNorm(g_l + y_l)
 *     h_out = h_{n_layers}
 * fdesc and adesc share d; the token type (fdesc) equals adesc->xtype.
 * layers: HOST array; head_idx [n_layers, n_heads] and head_counts [n_layers]
 * receive the head lists; idx [n_layers, C] and counts [n_layers] the FFN
 * lists; trace (optional) [n_layers, 2, B, d] in the token type receives each
 * layer's h_l and g_l.  h_out must not alias h_in.  Each layer appends its
 * listed heads' k and v at position len of its caches.
 */
PI_API pi_status pi_decode_blocks(const pi_ffn_desc *fdesc, const pi_attn_desc *adesc, int32_t batch,
                                  int32_t n_layers, const pi_block_weights *layers, const void *h_in, void *h_out,
                                  int32_t len, int32_t *head_idx, int32_t *head_counts, int32_t *idx,
                                  int32_t *counts, void *trace, float eps, void *ws, size_t ws_bytes, void *stream);

/*
 * pi_predict_static -- pi_predict for callers that cannot allocate device
 * memory.  The paper has no counterpart to this call; it exists for hosts
 * that hand the library only its inputs and outputs (plugin interfaces that
 * own every allocation, or serving loops that must not call cudaMalloc once
 * running, because an allocation can synchronise the device).
 *
 * Same arguments, argument checks and rules as pi_predict, minus the
 * workspace: the scratch lives in one library-owned device array of
 * PI_STATIC_SCRATCH_BYTES (1 MiB), held on every GPU that loads the library
 * until the process exits.  The list equals pi_predict's except for neurons
 * whose score lies within rounding (well under 1e-3) of the threshold: for
 * fp16 predictors and token blocks of 3-16 pi_predict runs its tensor-core
 * predictor, this call always the CUDA-core one.
 * Limit: align256(batch * rank * 4) + align256(ceil(C/256) * 32) +
 * align256(ceil(C/256) * 4) <= 1 MiB (C = ffn - n_hot), else
 * PI_ERR_CAPACITY and nothing is launched.  The call itself never calls
 * cudaMalloc.
 * - The first call on a device looks the array's address up on that device
 *   (cudaGetSymbolAddress).  Under CUDA's lazy module loading (the default)
 *   that first call may also load the library's device code on the device
 *   and create the array there, which can allocate and synchronise: make it
 *   during set-up, before any stream capture and before the loop that must
 *   not allocate (CUDA_MODULE_LOADING=EAGER loads it when the process starts).
 * - Every call shares the one array and the last call's contents stay in it;
 *   nothing in it needs to start at zero (each call writes all it reads).
 * - Calls that can overlap on the GPU (different streams, or several host
 *   threads) race on the array: order them on one stream.
 */
#define PI_STATIC_SCRATCH_BYTES ((size_t)1 << 20)
PI_API pi_status pi_predict_static(const pi_ffn_desc *desc, int32_t batch, const void *h, const void *P1,
                                   const void *P2, const float *bp, float threshold, int32_t *idx, int32_t *count,
                                   void *stream);

/*
 * pi_selftest_bounded_wait -- run one bounded wait that nothing will ever
 * satisfy, to exercise the failure path of the persistent kernel without a
 * GPU fault: kind 0 waits on a shared-memory mbarrier nobody arrives on,
 * kind 1 on a grid-barrier count nobody reaches.  The wait gives up after the
 * same limit the decode kernel uses (2 s), records PI_ERR_TIMEOUT in the
 * workspace status word, raises the workspace abort flag and returns; the
 * CUDA context stays usable.  Call pi_workspace_init before reusing `ws`.
 */
PI_API pi_status pi_selftest_bounded_wait(void *ws, int32_t kind, void *stream);

/* Text of the last host-side error in this thread (never NULL). */
PI_API const char *pi_last_error(void);

/* Library version, "major.minor.patch". */
PI_API const char *pi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PI_H_ */
