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
// One warp routes one token: lane r (< topk) returns the r-th chosen expert
// and its weight.
template <int VPL>  // logits per lane (E <= 32 * VPL)
__device__ __forceinline__ void route_token(const float* row, int E, int topk, int renormalize,
                                            int lane, int& out_id, float& out_w) {

  float v[VPL];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? (*(row + e)) : -INFINITY;
    if (e >= E) taken |= 1u << i;
  }
  // softmax statistics over all experts
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    if (!((taken >> i) & 1u)) m = fmaxf(m, v[i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float z = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    if (!((taken >> i) & 1u)) z += expf(v[i] - m);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);

  // k rounds of warp argmax; lane r keeps the r-th choice
  float my_logit = 0.f;
  int my_id = -1;
  for (int r = 0; r < topk; ++r) {
    float best = -INFINITY;
    int bi = INT_MAX;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if ((taken >> i) & 1u) continue;
      if (bi == INT_MAX || v[i] > best) {  // ascending index inside a lane: strict > keeps the lower one
        best = v[i];
        bi = lane + 32 * i;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (oi != INT_MAX && (bi == INT_MAX || ob > best || (ob == best && oi < bi))) {
        best = ob;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == r) {
      my_logit = best;
      my_id = bi;
    }
  }
  const float ex = (lane < topk) ? expf(my_logit - m) : 0.f;
  float s = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  out_id = my_id;
  out_w = renormalize ? __fdiv_rn(ex, s) : __fdiv_rn(ex, z);
}

}  // namespace moe
