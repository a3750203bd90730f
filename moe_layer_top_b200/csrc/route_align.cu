// Router and expert alignment kernels.
//
// Router ("Warum MoE-Kernel so wichtig sind", AWS/kinachrichten page: token
// routing): one warp per token, the E logits spread over the lanes; k rounds
// of a warp-wide argmax pick the experts (descending logit, lower index on
// ties); softmax statistics come from butterfly reductions, so the result is
// bitwise reproducible.
//
// Alignment (vLLM PR #64760 analysis, §1.1: sorted_token_ids,
// num_tokens_post_padded, BLOCK_SIZE_M-padded expert runs): a counting sort
// of the flat assignments t*topk + j by expert in three passes --
//   1. per warp-chunk of 256 assignments, an expert histogram (shared-memory
//      atomics; counts are order independent);
//   2. per expert, an exclusive scan of its chunk counts (chunk order);
//   3. per warp-chunk, a stable scatter: the rank of an assignment among the
//      earlier ones of its expert inside the chunk comes from __match_any_sync
//      over 32 lanes plus a per-warp running counter, so the sorted order is
//      ascending flat order inside every expert, whatever the scheduling.
// Padding slots, the tail past num_tokens_post_padded and the per-block
// expert ids are filled by the same third pass.
//
// Expert parallelism ("Hosting von Qwen auf Blackwell", "Experten-Parallel":
// the dispatch picks the tokens routed to this rank's experts): the router
// scores all experts and the ids stay global; the alignment keeps only the
// assignments to the local range [first, first + E), which it renumbers from
// zero, so every later stage sees an ordinary E-expert problem.
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "router.cuh"

namespace moe {

template <int VPL>
__global__ void __launch_bounds__(256) route_kernel(const float* logits, int T, int E, int topk,
                                                    int renormalize, int32_t* ids,
                                                    float* weights) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int tok = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (tok >= T) return;
  int id;
  float w;
  route_token<VPL>(logits + static_cast<size_t>(tok) * E, E, topk, renormalize, lane, id, w);
  if (lane < topk) {
    const size_t o = static_cast<size_t>(tok) * topk + lane;
    ids[o] = id;
    weights[o] = w;
  }
}

cudaError_t launch_route(const float* logits, int T, int E, int topk, int renormalize, int32_t* ids,
                         float* weights, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int threads = 256;
  const int blocks = static_cast<int>((static_cast<long long>(T) * 32 + threads - 1) / threads);
  if (E <= 128)
    return launch_pdl(route_kernel<4>, blocks, threads, 0, stream, logits, T, E, topk, renormalize, ids, weights);
  if (E <= 256)
    return launch_pdl(route_kernel<8>, blocks, threads, 0, stream, logits, T, E, topk, renormalize, ids, weights);
  if (E <= 512)
    return launch_pdl(route_kernel<16>, blocks, threads, 0, stream, logits, T, E, topk, renormalize, ids, weights);
  return launch_pdl(route_kernel<32>, blocks, threads, 0, stream, logits, T, E, topk, renormalize, ids, weights);
}

// ----------------------------------------------------------------------------
// align pass 1: per-chunk expert histograms
// ----------------------------------------------------------------------------
constexpr int kAlignWarps = 8;

__global__ void __launch_bounds__(kAlignWarps * 32) align_count_kernel(const int32_t* ids, int n,
                                                                       int E, ExpertRange er, int nchunks,
                                                                       int32_t* chunk_counts,
                                                                       int* status) {
  extern __shared__ int32_t hist_all[];
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * kAlignWarps + warp;
  if (chunk >= nchunks) return;
  int32_t* hist = hist_all + warp * E;
  for (int e = lane; e < E; e += 32) hist[e] = 0;
  __syncwarp();
  const int base = chunk * kAlignChunk;
  for (int i = lane; i < kAlignChunk; i += 32) {
    const int f = base + i;
    if (f < n) {
      const int g = (*(ids + f));
      const int e = g - er.first;
      if (g < 0 || g >= er.e_global)
        report_status(status, MOE_STATUS_BAD_EXPERT_ID);
      else if (e >= 0 && e < E)
        atomicAdd(&hist[e], 1);  // other ranks' experts are not counted here
    }
  }
  __syncwarp();
  int32_t* out = chunk_counts + static_cast<size_t>(chunk) * E;
  for (int e = lane; e < E; e += 32) out[e] = hist[e];
}

// ----------------------------------------------------------------------------
// align pass 2: per expert, exclusive scan over chunks (in place) and total
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) align_scan_kernel(int32_t* chunk_counts, int nchunks, int E,
                                                         int32_t* counts_ws,
                                                         int32_t* user_counts) {
  __shared__ int32_t warp_sums[8];
  pdl_launch_dependents();
  pdl_wait();
  const int e = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t carry = 0;
  for (int c0 = 0; c0 < nchunks; c0 += 256) {
    const int c = c0 + threadIdx.x;
    const int32_t v = (c < nchunks) ? chunk_counts[static_cast<size_t>(c) * E + e] : 0;
    int32_t incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int32_t before = 0, tile_total = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const int32_t s = warp_sums[w];
      if (w < warp) before += s;
      tile_total += s;
    }
    if (c < nchunks) chunk_counts[static_cast<size_t>(c) * E + e] = carry + before + incl - v;
    carry += tile_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    counts_ws[e] = carry;
    if (user_counts) user_counts[e] = carry;
  }
}

// ----------------------------------------------------------------------------
// align pass 3: stable scatter, padding, block expert ids
// ----------------------------------------------------------------------------
__device__ __forceinline__ int owner_expert(const int32_t* offs, int E, int p) {
  // largest e with offs[e] <= p (offs non-decreasing, offs[0] = 0)
  int lo = 0, hi = E;  // invariant: offs[lo] <= p, answer in [lo, hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offs[mid] <= p)
      lo = mid;
    else
      hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kAlignWarps * 32) align_scatter_kernel(
    const int32_t* ids, int n, int E, int first, int block_m, int capacity, int nchunks,
    const int32_t* chunk_base, const int32_t* counts_ws, int32_t* sorted_ids,
    int32_t* expert_ids, int32_t* ntpp_out, int32_t* offsets_ws,
    int32_t* user_offsets, int32_t* pos_of_flat) {
  extern __shared__ int32_t smem_i32[];
  int32_t* offs = smem_i32;                    // [E + 1]
  int32_t* cnt = offs + (E + 1);               // [E]
  int32_t* running = cnt + E;                  // [kAlignWarps][E]
  __shared__ int32_t warp_sums[kAlignWarps];
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // padded offsets: exclusive scan of round_up(count, block_m) over experts
  int32_t carry = 0;
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    const int32_t c = (e < E) ? counts_ws[e] : 0;
    if (e < E) cnt[e] = c;
    const int32_t v = (c + block_m - 1) / block_m * block_m;
    int32_t incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int32_t before = 0, tile_total = 0;
    for (int w = 0; w < kAlignWarps; ++w) {
      const int32_t s = warp_sums[w];
      if (w < warp) before += s;
      tile_total += s;
    }
    if (e < E) offs[e] = carry + before + incl - v;
    carry += tile_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) offs[E] = carry;
  __syncthreads();
  const int ntpp = offs[E];
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e <= E; e += blockDim.x) {
      offsets_ws[e] = offs[e];
      if (user_offsets) user_offsets[e] = offs[e];
    }
    if (threadIdx.x == 0) *ntpp_out = ntpp;
  }

  // stable scatter of this block's warp-chunks
  const int chunk = blockIdx.x * kAlignWarps + warp;
  if (chunk < nchunks) {
    int32_t* run = running + warp * E;
    for (int e = lane; e < E; e += 32) run[e] = 0;
    __syncwarp();
    const int32_t* cb = chunk_base + static_cast<size_t>(chunk) * E;
    const int base = chunk * kAlignChunk;
    for (int i0 = 0; i0 < kAlignChunk; i0 += 32) {
      const int f = base + i0 + lane;
      int e = -1;
      if (f < n) {
        e = (*(ids + f)) - first;
        if (e < 0 || e >= E) e = -1;  // invalid (reported by pass 1) or not local: never indexed
      }
      const uint32_t same = __match_any_sync(0xffffffffu, e);
      const uint32_t lower = same & ((1u << lane) - 1u);
      const int rank = __popc(lower);
      int dest = -1;
      if (e >= 0) dest = offs[e] + cb[e] + run[e] + rank;
      __syncwarp();
      if (e >= 0) {
        sorted_ids[dest] = f;
        if (lower == 0) run[e] += __popc(same);  // one lane per expert group updates the counter
      }
      if (pos_of_flat && f < n) pos_of_flat[f] = dest;  // -1 for an invalid id
      __syncwarp();
    }
  }

  // sentinel in padding and tail; expert of every block
  const int stride = gridDim.x * blockDim.x;
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < capacity; p += stride) {
    bool pad = true;
    if (p < ntpp) {
      const int e = owner_expert(offs, E, p);
      pad = p >= offs[e] + cnt[e];
    }
    if (pad) sorted_ids[p] = n;
  }
  const int nblocks = capacity / block_m;
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
    const int p = b * block_m;
    expert_ids[b] = (p < ntpp) ? owner_expert(offs, E, p) : -1;
  }
}

cudaError_t launch_align(const int32_t* topk_ids, int n, int E, ExpertRange er, int block_m, int capacity,
                         int32_t* sorted_ids,
                         int32_t* expert_ids, int32_t* ntpp, int32_t* counts_ws, int32_t* offsets_ws,
                         int32_t* chunk_scratch, int32_t* user_counts, int32_t* user_offsets, int* status,
                         int32_t* pos_of_flat, cudaStream_t stream) {
  const int nchunks = align_chunks(n);
  if (nchunks == 0) return cudaSuccess;
  const int threads = kAlignWarps * 32;
  const int blocks = (nchunks + kAlignWarps - 1) / kAlignWarps;
  const size_t smem1 = static_cast<size_t>(kAlignWarps) * E * sizeof(int32_t);
  cudaError_t err = launch_pdl(align_count_kernel, blocks, threads, smem1, stream, topk_ids, n, E, er, nchunks,
                               chunk_scratch, status);
  if (err != cudaSuccess) return err;
  err = launch_pdl(align_scan_kernel, E, 256, 0, stream, chunk_scratch, nchunks, E, counts_ws, user_counts);
  if (err != cudaSuccess) return err;
  const size_t smem3 = (static_cast<size_t>(E + 1) + E + static_cast<size_t>(kAlignWarps) * E) * sizeof(int32_t);
  int blocks3 = blocks;
  const int fill_blocks = (capacity + threads * 4 - 1) / (threads * 4);
  if (fill_blocks > blocks3) blocks3 = fill_blocks < 296 ? fill_blocks : 296;
  if (blocks3 < blocks) blocks3 = blocks;
  return launch_pdl(align_scatter_kernel, blocks3, threads, smem3, stream, topk_ids, n, E, er.first, block_m, capacity,
                    nchunks, chunk_scratch, counts_ws, sorted_ids, expert_ids, ntpp, offsets_ws, user_offsets,
                    pos_of_flat);
}

// ----------------------------------------------------------------------------
// Small batches: routing and the whole alignment in one CTA of 1024 threads.
// The assignments are split into 32 contiguous warp-chunks; per-warp expert
// histograms, a per-expert scan over the warps, a block scan of the padded
// counts, then each warp scatters its chunk in order (ranks from
// __match_any_sync plus a running per-warp base), which is the same stable
// order as the multi-CTA path.
// ----------------------------------------------------------------------------
template <int VPL>
__global__ void __launch_bounds__(1024) route_align_small_kernel(
    const float* logits, const int32_t* ids_in, int T, int E, ExpertRange er, int topk, int renormalize,
    int32_t* ids_out, float* weights_out, int block_m, int capacity,
    int32_t* sorted_ids, int32_t* expert_ids, int32_t* ntpp_out,
    int32_t* counts_out, int32_t* offsets_out, int* status, int32_t* pos_of_flat) {
  extern __shared__ int32_t sm_small[];
  __shared__ int32_t warp_sums[32];
  pdl_launch_dependents();
  pdl_wait();
  const int n = T * topk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* ids_s = sm_small;           // [n]
  int32_t* hist = ids_s + n;           // [32][E]: counts, then running bases
  int32_t* offs = hist + 32 * E;       // [E + 1]
  int32_t* cnt = offs + E + 1;         // [E]

  if (logits != nullptr) {
    // each warp routes tokens warp, warp + 32, ...; the next token's logits are loaded while the
    // current one is routed
    float cur[VPL], nxt[VPL];
    if (warp < T) load_logits<VPL>(logits + static_cast<size_t>(warp) * er.e_global, er.e_global, lane, cur);
    for (int t = warp; t < T; t += 32) {
      if (t + 32 < T) load_logits<VPL>(logits + static_cast<size_t>(t + 32) * er.e_global, er.e_global, lane, nxt);
      int id;
      float w;
      route_token_vals<VPL>(cur, er.e_global, topk, renormalize, lane, id, w);
      if (lane < topk) {
        ids_out[t * topk + lane] = id;
        weights_out[t * topk + lane] = w;
        ids_s[t * topk + lane] = id;
      }
#pragma unroll
      for (int i = 0; i < VPL; ++i) cur[i] = nxt[i];
    }
  } else {
    for (int i = tid; i < n; i += 1024) ids_s[i] = (*(ids_in + i));
  }
  const int chunk = (n + 32 * 32 - 1) / (32 * 32) * 32;  // multiple of 32
  const int nw = (n + chunk - 1) / chunk;                 // warps that own assignments
  const int begin = warp * chunk;
  const int end = min(begin + chunk, n);
  for (int i = tid; i < nw * E; i += 1024) hist[i] = 0;
  __syncthreads();

  for (int i = begin + lane; i < end; i += 32) {
    const int g = ids_s[i];
    const int e = g - er.first;
    if (g < 0 || g >= er.e_global)
      report_status(status, MOE_STATUS_BAD_EXPERT_ID);
    else if (e >= 0 && e < E)
      atomicAdd(&hist[warp * E + e], 1);
  }
  __syncthreads();
  for (int e = tid; e < E; e += 1024) {
    int32_t run = 0;
    for (int w = 0; w < nw; ++w) {
      const int32_t v = hist[w * E + e];
      hist[w * E + e] = run;
      run += v;
    }
    cnt[e] = run;
  }
  __syncthreads();
  {
    const int32_t v = tid < E ? (cnt[tid] + block_m - 1) / block_m * block_m : 0;
    int32_t incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    // only the first ceil(E / 32) warps hold experts (E <= 256): a thread adds the sums of
    // the warps before its own, thread 0 all of them
    if (tid < E) {
      int32_t before = 0;
      for (int w = 0; w < warp; ++w) before += warp_sums[w];
      offs[tid] = before + incl - v;
    }
    if (tid == 0) {
      int32_t total = 0;
      for (int w = 0; w < (E + 31) / 32; ++w) total += warp_sums[w];
      offs[E] = total;
    }
  }
  __syncthreads();
  const int ntpp = offs[E];

  for (int i0 = begin; i0 < end; i0 += 32) {
    const int i = i0 + lane;
    int e = -1;
    if (i < end) {
      e = ids_s[i] - er.first;
      if (e < 0 || e >= E) e = -1;  // invalid or not local
    }
    const uint32_t same = __match_any_sync(0xffffffffu, e);
    const uint32_t lower = same & ((1u << lane) - 1u);
    int dest = -1;
    if (e >= 0) dest = offs[e] + hist[warp * E + e] + __popc(lower);
    __syncwarp();
    if (e >= 0) {
      sorted_ids[dest] = i;
      if (lower == 0) hist[warp * E + e] += __popc(same);
    }
    if (pos_of_flat && i < end) pos_of_flat[i] = dest;  // -1 for an invalid id
    __syncwarp();
  }
  // padding: each expert's slots past its count (one warp per expert, consecutive lanes on
  // consecutive slots), then everything past num_tokens_post_padded; block experts: each
  // expert's blocks, then -1 past the used ones
  for (int e = warp; e < E; e += 32) {
    const int p1 = offs[e + 1];
    for (int p = offs[e] + cnt[e] + lane; p < p1; p += 32) sorted_ids[p] = n;
    for (int b = offs[e] / block_m + lane; b < p1 / block_m; b += 32) expert_ids[b] = e;
  }
  for (int p = ntpp + tid; p < capacity; p += 1024) sorted_ids[p] = n;
  for (int b = ntpp / block_m + tid; b < capacity / block_m; b += 1024) expert_ids[b] = -1;
  for (int e = tid; e <= E; e += 1024) {
    offsets_out[e] = offs[e];
    if (e < E) counts_out[e] = cnt[e];
  }
  if (tid == 0) *ntpp_out = ntpp;
}

bool route_align_small_fits(long long n, int e_global) {
  return n > 0 && n <= kSmallAlignMaxN && e_global <= kSmallAlignMaxE;
}

cudaError_t launch_route_align_small(const float* logits, const int32_t* ids_in, int T, int E, ExpertRange er,
                                     int topk, int renormalize, int32_t* ids_out, float* weights_out, int block_m,
                                     int capacity, int32_t* sorted_ids, int32_t* expert_ids, int32_t* ntpp,
                                     int32_t* counts, int32_t* offsets, int* status, int32_t* pos_of_flat,
                                     cudaStream_t stream) {
  const size_t smem = (static_cast<size_t>(T) * topk + 32 * static_cast<size_t>(E) + 2 * static_cast<size_t>(E) + 1) *
                      sizeof(int32_t);
  static bool attr_set[4] = {false, false, false, false};
  auto pick = [&](auto kern, int idx) -> cudaError_t {
    if (!attr_set[idx]) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
      if (e != cudaSuccess) return e;
      attr_set[idx] = true;
    }
    return launch_pdl(kern, 1, 1024, smem, stream, logits, ids_in, T, E, er, topk, renormalize, ids_out,
                      weights_out, block_m, capacity, sorted_ids, expert_ids, ntpp, counts, offsets, status,
                      pos_of_flat);
  };
  if (er.e_global <= 128) return pick(route_align_small_kernel<4>, 0);
  return pick(route_align_small_kernel<8>, 1);
}

}  // namespace moe
