// pi_layout.h -- byte layout of a libpi workspace (host side).
//
//   [ctrl 2304 B: status, abort, barrier count and base, claim and hand-over counters]
//   [u: B x rank fp32][tile masks][tile counts][a: B x ffn fp32]
//   [partials: G_MAX x B x d fp32][y: B x d fp32][h: B x d fp32]
//   [y accumulators][list counts: 128 x G_MAX][handed-over cold rows: 128 x C]
//   [pre-activations of the tensor-core token-block path: 4 x (ffn + 16) x 2 x B fp32,
//    token blocks of 3 or more only]
//   [scratch of the tcgen05 token-block FFN (tc_ws_bytes), token blocks of 3 or more only]
//
// Every region starts on a 256-byte boundary.  The layout depends only on the
// descriptor and the batch, never on the device.
#pragma once
#include <stddef.h>
#include <stdint.h>

namespace pi {

// workspace bytes of the tcgen05 token-block FFN (pi_tc.cu)
size_t tc_ws_bytes(int d, int ffn, int B);

constexpr int kGMax = 296;  // split-K partial slots (2 x 148 SMs)
#ifndef PI_YCOPIES
#define PI_YCOPIES 1
#endif
constexpr int kYAccCopies = PI_YCOPIES;  // copies of the persistent kernel's fp32 output accumulator
constexpr int kLayersMax = 128;  // layers of one decode-stack call
constexpr size_t kCtrlBytes = 2304;  // the control block at the start of a workspace

struct WsLayout {
  size_t u, tile_mask, tile_count, act, partial, ybuf, hbuf, yacc, lcnt, don, pre, tc, total;
  int n_tiles, g_max;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

inline WsLayout ws_layout(int d, int ffn, int n_hot, int rank, int B) {
  WsLayout L;
  size_t off = kCtrlBytes;
  const int C = ffn - n_hot;
  L.n_tiles = (C + 255) / 256;
  L.g_max = kGMax;
  L.u = off; off += align256((size_t)B * rank * 4);
  L.tile_mask = off; off += align256((size_t)(L.n_tiles > 0 ? L.n_tiles : 1) * 8 * 4);
  L.tile_count = off; off += align256((size_t)(L.n_tiles > 0 ? L.n_tiles : 1) * 4);
  L.act = off; off += align256((size_t)B * ffn * 4);
  L.partial = off; off += align256((size_t)kGMax * B * d * 4);
  L.ybuf = off; off += align256((size_t)B * d * 4);
  L.hbuf = off; off += align256((size_t)B * d * 4);
  L.yacc = off; off += align256((size_t)2 * kYAccCopies * B * d * 4);
  L.lcnt = off; off += align256((size_t)kLayersMax * kGMax * 4);
  L.don = off; off += align256((size_t)kLayersMax * (C > 0 ? C : 1) * 4);
  L.pre = off; off += B >= 3 ? align256((size_t)4 * ((ffn + 17) & ~1) * 2 * B * 4) : 0;
  L.tc = off; off += B >= 3 ? align256(tc_ws_bytes(d, ffn, B)) : 0;
  L.total = off;
  return L;
}

}  // namespace pi
