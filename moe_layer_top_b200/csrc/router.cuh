// Router device function shared by the routing kernels and the persistent
// decode kernel ("Warum MoE-Kernel so wichtig sind", AWS/kinachrichten page:
// token routing).  One warp routes one token; see route_align.cu.
#pragma once

#include <climits>

#include "common.cuh"

namespace moe {

// ----------------------------------------------------------------------------
// router
// ----------------------------------------------------------------------------
// Order-preserving 32-bit key of a finite float (larger float -> larger key;
// -0 is folded onto +0 first so that equal logits get equal keys); 0 is below
// every key and marks "taken / no expert".
__device__ __forceinline__ uint32_t logit_key(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// One warp routes one token (route_token_vals: logits already loaded by
// load_logits): lane r (< topk) returns the r-th chosen expert and its
// weight.  Each selection round is two warp reductions (redux.sync):
// the largest key, then the lowest expert index holding it -- descending
// logit, the lower index on ties.
// This lane's logits of one token: expert lane + 32 i in v[i] (-inf past E).
template <int VPL>
__device__ __forceinline__ void load_logits(const float* row, int E, int lane, float (&v)[VPL]) {
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? (*(row + e)) : -INFINITY;
  }
}

template <int VPL>  // logits per lane (E <= 32 * VPL), already in registers
__device__ __forceinline__ void route_token_vals(const float (&v)[VPL], int E, int topk, int renormalize,
                                                 int lane, int& out_id, float& out_w) {
  uint32_t key[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) key[i] = (lane + 32 * i < E) ? logit_key(v[i]) : 0u;
  // softmax statistics over all experts
  uint32_t kmax = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) kmax = max(kmax, key[i]);
  const float m = key_logit(__reduce_max_sync(0xffffffffu, kmax));
  float z = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    if (lane + 32 * i < E) z += expf(v[i] - m);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);

  // k rounds of warp argmax; lane r keeps the r-th choice
  float my_logit = 0.f;
  int my_id = -1;
  for (int r = 0; r < topk; ++r) {
    uint32_t best = 0;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (key[i] > best) {  // ascending index inside a lane: strict > keeps the lower one
        best = key[i];
        bi = i;
      }
    const uint32_t wbest = __reduce_max_sync(0xffffffffu, best);
    const uint32_t cand = (best == wbest) ? static_cast<uint32_t>(lane + 32 * bi) : 0xffffffffu;
    const int widx = static_cast<int>(__reduce_min_sync(0xffffffffu, cand));
    if ((widx & 31) == lane) {
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (i == (widx >> 5)) key[i] = 0u;
    }
    if (lane == r) {
      my_logit = key_logit(wbest);
      my_id = widx;
    }
  }
  const float ex = (lane < topk) ? expf(my_logit - m) : 0.f;
  float s = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  out_id = my_id;
  out_w = renormalize ? __fdiv_rn(ex, s) : __fdiv_rn(ex, z);
}

template <int VPL>
__device__ __forceinline__ void route_token(const float* row, int E, int topk, int renormalize,
                                            int lane, int& out_id, float& out_w) {
  float v[VPL];
  load_logits<VPL>(row, E, lane, v);
  route_token_vals<VPL>(v, E, topk, renormalize, lane, out_id, out_w);
}

}  // namespace moe
