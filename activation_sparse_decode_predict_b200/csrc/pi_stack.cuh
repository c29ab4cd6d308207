// pi_stack.cuh -- parameters and launcher of the persistent decode-step kernel.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pi_common.cuh"

namespace pi {

constexpr int kMaxLayers = 128;
constexpr int kMaxDevices = 64;      // devices per process the launcher keeps state for
constexpr int kTraceEvents = 16;     // phase stamps per (layer, CTA) of a PI_TRACE build
constexpr int kNQ = 64;              // items in flight per CTA (queue depth)
constexpr int kMaxConsumers = 512;   // consumer threads per CTA (d <= 8192)
constexpr int kMaxRank = 4096;
constexpr size_t kSmemBytes = 232448;  // opt-in shared memory per CTA on sm_100
#ifndef PI_YCOPIES
#define PI_YCOPIES 1
#endif
#ifndef PI_HOT_A
#define PI_HOT_A 0
#endif
#ifndef PI_HOT_B
#define PI_HOT_B 0
#endif
#ifndef PI_STACK_EPT_MIN
#define PI_STACK_EPT_MIN 8
#endif
constexpr int kYCopies = PI_YCOPIES;  // fp32 output accumulator copies (spreads the atomics)
// static hot neurons per CTA before barrier U (A) and at the head of the
// neuron stream (B); 0 means one neuron group
constexpr int kHotA = PI_HOT_A, kHotB = PI_HOT_B;
constexpr int kEptMin = PI_STACK_EPT_MIN;  // columns of d per consumer thread (8 or 16)
#ifndef PI_DONATE
#define PI_DONATE 1
#endif
constexpr int kDonate = PI_DONATE;  // 1: a CTA hands excess predicted rows to the other CTAs
#ifndef PI_F16_MMA
#define PI_F16_MMA 0
#endif
#ifndef PI_MMA_X2
#define PI_MMA_X2 0
#endif
#ifndef PI_P1_MMA
#define PI_P1_MMA 0
#endif
// fp16 predictors: the P1 dots of a single token run on CUDA cores (one token
// fills 1 of the 8 columns of the tensor-core operand); 1 puts them on the
// tensor cores too.  Token blocks of 2 always use the tensor cores.
constexpr bool kP1Mma = PI_P1_MMA != 0;
constexpr bool kF16Mma = PI_F16_MMA != 0;  // fp16 neuron groups: gate/up dots on the tensor cores
constexpr bool kMmaX2 = PI_MMA_X2 != 0;    // load only tile rows 0-7 when a group fills no more
#ifndef PI_NG_FULL
#define PI_NG_FULL 0
#endif
constexpr int kNgFull = PI_NG_FULL;  // 1: groups may fill the ring but one item (else half the ring)
#ifndef PI_LAZY_TAIL
#define PI_LAZY_TAIL 0
#endif
#ifndef PI_TAIL_GROUPS
#define PI_TAIL_GROUPS 1
#endif
// 1: the last claims of a layer wait until the CTA's own queue holds at most
// kTailGroups neuron groups
constexpr bool kLazyTail = PI_LAZY_TAIL != 0;
constexpr int kTailGroups = PI_TAIL_GROUPS;
constexpr int kGMaxCtas = 296;       // largest grid (2 x 148)
constexpr int kShareRegs = 2;        // per-thread registers for the CTA's bias shares
constexpr int kMaxKQ = 4;            // k-parts of a P2 tile at most (each has its own score slot)
constexpr int kMaxGroup = 16;        // neurons per group at most

// One layer's device pointers (a copy of pi_layer_weights).
struct StackLayer {
  const void* P1;
  const void* P2;
  const float* bp;
  const void* wg;
  const void* wg_sc;
  const void* wu;
  const void* wu_sc;
  const void* wd;
  const void* wd_sc;
  const float* b1;
  const float* b2;
  const void* P1_sc;  // Q4_0 predictors: scales of P1 [rank, d/32] and P2 [C, rank/32] (else null)
  const void* P2_sc;
  float thr;
  int rank;           // this layer's predictor rank (<= the descriptor's)
};

struct StackParams {
  int d, ffn, n_hot, rank, act, L;
  float eps;
  int T;           // consumer threads (d / stack_ept(d))
  int ring_bytes;  // shared-memory ring size
  int seg_cap;     // per-CTA capacity of the local active lists
  int ng;          // neurons per group (<= 4 on CUDA cores; one 16-row tile with PI_F16_MMA)
  int p1rows;      // P1 rows per tensor-core group (fp16 predictors)
  int hot_a;       // hot neurons [0, hot_a) are shared out statically, consumed before barrier U
  int hot_static;  // [hot_a, hot_static) are shared out statically, at the head of the neuron
                   // stream; the rest, [hot_static, n_hot), are claimed
  int don_slack;   // a CTA keeps its predicted cold rows up to its running mean + don_slack
  int cmp_layers;  // layers per chunk of the final list compaction
  int off_bars, off_itemoff, off_u, off_bp, off_cidx, off_act, off_red, off_gred, off_misc;
  int off_hb, off_ub, off_zero, off_redp, off_sc;
  const void* h_in;
  void* h_out;
  int32_t* idx;     // [L, C]
  int32_t* counts;  // [L]
  float* y_out;     // [L, B, d] or null
  void* h_trace;    // [L, B, d] or null
  Ctrl* ctrl;
  float* u_g;       // [B, r]
  float* yacc;      // [2, kYCopies, B, d] fp32 output accumulators
  int* pool;        // [L] claim counters of the hot neurons (zero between launches)
  int* lcnt;        // [L, G] per-CTA counts of the local active lists
  int* don;         // [L, C] cold rows handed to other CTAs (row + 1; zero = not written yet)
  uint64_t* trace;  // [L, G, kTraceEvents] phase stamps (PI_TRACE builds only; else unused)
  StackLayer layers[kMaxLayers];
};

// Whether the kernel keeps the token block as fp16 rows in shared memory (the
// tensor-core operand of the P1 dots of a token block of 2, or of tensor-core
// neuron groups).
__host__ __device__ constexpr bool stack_token_rows(int ptype, int B) {
  return ptype == kF16 && (B > 1 || kP1Mma || kF16Mma);
}

// Whether a layer of this predictor rank fits the kernel: fp16 predictors feed
// the tensor cores in 16-element steps; Q4_0 predictor rows go to shared
// memory as whole rows of codes and of scales, 16-byte multiples when the
// rank is a multiple of 256.
__host__ __device__ constexpr bool stack_rank_ok(int ptype, int rank) {
  return rank > 0 && rank <= kMaxRank && (ptype == kF16 ? rank % 16 == 0 : ptype == kQ4_0 ? rank % 256 == 0 : rank % 8 == 0);
}

// Columns of d each consumer thread owns (8 when d/8 threads fit, else 16).
int stack_ept(int d);
bool stack_supported(int wtype, int ptype, int d, int ffn, int n_hot, int rank, int B, int L);
// Fills the shared-memory offsets of p (needs d, ffn, n_hot, rank); returns the
// dynamic shared memory size, or 0 if it does not fit.
size_t stack_smem_layout(StackParams& p, int ptype, int B, int G);
cudaError_t launch_stack(int wtype, int ptype, int B, const StackParams& p, int G, size_t smem, cudaStream_t st);

}  // namespace pi
