// C ABI of the fused MoE layer: argument validation, problem resolution,
// workspace layout and the stage pipeline.  Every entry point validates all
// of its arguments before it enqueues anything.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "allreduce.h"
#include "kernels.h"
#include "moe_b200.h"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;

// Streaming multiprocessor count of the current device, and whether it is an
// sm_100 part (the only architecture this library is built for).
int device_check(int* sms) {
  static int cache_sms[kMaxDevices] = {0};
  static int cache_ok[kMaxDevices] = {0};  // 0 unknown, 1 ok, -1 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device index %d out of range", dev);
  if (cache_ok[dev] == 0) {
    int major = 0, minor = 0, n = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    cache_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
    cache_sms[dev] = n;
    if (cache_ok[dev] < 0)
      return fail(MOE_ERR_UNSUPPORTED, "compute capability %d.%d: this library runs on sm_100 (B200) only", major,
                  minor);
  }
  if (cache_ok[dev] < 0) return fail(MOE_ERR_UNSUPPORTED, "this library runs on sm_100 (B200) only");
  if (sms) *sms = cache_sms[dev];
  return MOE_OK;
}

inline int64_t align256(int64_t v) { return (v + 255) & ~int64_t(255); }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Router width: every expert, of which this call holds [first_expert, first_expert + E).
int global_experts(const moe_problem* p) { return p->num_global_experts == 0 ? p->E : p->num_global_experts; }

bool expert_parallel(const moe_problem* p) { return global_experts(p) != p->E; }

int validate_problem(const moe_problem* p) {
  if (p == nullptr) return fail(MOE_ERR_INVALID, "problem is NULL");
  if (p->T < 0) return fail(MOE_ERR_INVALID, "T = %d < 0", p->T);
  if (p->E < 1 || p->E > 1024) return fail(MOE_ERR_INVALID, "E = %d outside [1, 1024]", p->E);
  if (p->num_global_experts != 0 && (p->num_global_experts < p->E || p->num_global_experts > 1024))
    return fail(MOE_ERR_INVALID, "num_global_experts = %d outside [E, 1024] (E = %d; 0 = E)", p->num_global_experts,
                p->E);
  if (p->first_expert < 0 || p->first_expert > global_experts(p) - p->E)
    return fail(MOE_ERR_INVALID, "first_expert = %d outside [0, num_global_experts - E] = [0, %d]", p->first_expert,
                global_experts(p) - p->E);
  if (p->topk < 1 || p->topk > global_experts(p) || p->topk > 32)
    return fail(MOE_ERR_INVALID, "topk = %d outside [1, min(num_global_experts, 32)]", p->topk);
  if (p->H <= 0 || p->H % 128) return fail(MOE_ERR_INVALID, "H = %d is not a positive multiple of 128", p->H);
  if (p->I <= 0 || p->I % 128) return fail(MOE_ERR_INVALID, "I = %d is not a positive multiple of 128", p->I);
  if (static_cast<int64_t>(p->T) * p->topk >= (int64_t(1) << 31))
    return fail(MOE_ERR_INVALID, "T * topk overflows int32");
  if (static_cast<int64_t>(p->E) * 2 * p->I >= (int64_t(1) << 31) ||
      static_cast<int64_t>(p->E) * p->H >= (int64_t(1) << 31))
    return fail(MOE_ERR_INVALID, "E * 2I or E * H overflows int32");
  if (p->weight_dtype != MOE_DTYPE_BF16 && p->weight_dtype != MOE_DTYPE_FP8_E4M3 &&
      p->weight_dtype != MOE_DTYPE_MXFP8_E4M3)
    return fail(MOE_ERR_UNSUPPORTED, "weight_dtype %d", p->weight_dtype);
  if (p->mode < MOE_MODE_AUTO || p->mode > MOE_MODE_SWAP_AB) return fail(MOE_ERR_INVALID, "mode %d", p->mode);
  if (p->renormalize != 0 && p->renormalize != 1) return fail(MOE_ERR_INVALID, "renormalize must be 0 or 1");
  if (p->split_k != 0 && p->split_k != 1) return fail(MOE_ERR_INVALID, "split_k must be 0 or 1");
  if (p->reserved[0] != 0) return fail(MOE_ERR_INVALID, "reserved fields must be zero");
  if (p->persistent_decode != 0 && p->persistent_decode != 1)
    return fail(MOE_ERR_INVALID, "persistent_decode must be 0 or 1");
  if (p->router_weight_on_input != 0 && p->router_weight_on_input != 1)
    return fail(MOE_ERR_INVALID, "router_weight_on_input must be 0 or 1");
  if (p->router_weight_on_input == 1 && p->topk != 1)
    return fail(MOE_ERR_INVALID, "router_weight_on_input needs topk == 1 (got %d)", p->topk);
  if (!(p->swiglu_limit >= 0.0f) || p->swiglu_limit == INFINITY)
    return fail(MOE_ERR_INVALID, "swiglu_limit must be 0 (off) or a positive finite value");
  const bool fp8 = p->weight_dtype == MOE_DTYPE_FP8_E4M3;
  // normal tiles cover 256 output columns of GEMM2 at a time
  if ((p->mode == MOE_MODE_NORMAL || (p->mode == MOE_MODE_AUTO && p->block_m >= 128)) && p->H % 256)
    return fail(MOE_ERR_INVALID, "normal tiles need H %% 256 == 0 (H = %d); use swap-AB", p->H);
  if (p->weight_dtype == MOE_DTYPE_MXFP8_E4M3) {
    if (p->mode == MOE_MODE_SWAP_AB) return fail(MOE_ERR_UNSUPPORTED, "MXFP8 weights run normal tiles only");
    if (p->H % 256) return fail(MOE_ERR_UNSUPPORTED, "MXFP8 weights need H %% 256 == 0 (H = %d)", p->H);
    if (p->block_m != 0 && p->block_m != 128)
      return fail(MOE_ERR_INVALID, "MXFP8 weights use block_m = 128 (got %d)", p->block_m);
  }
  if (p->mode == MOE_MODE_NORMAL && p->block_m != 0 && p->block_m != 128)
    return fail(MOE_ERR_INVALID, "normal mode uses block_m = 128 (got %d)", p->block_m);
  if (p->mode == MOE_MODE_SWAP_AB && p->block_m != 0 && p->block_m != 16 && p->block_m != 32 && p->block_m != 64)
    return fail(MOE_ERR_INVALID, "swap-AB mode uses block_m in {16, 32, 64} (got %d)", p->block_m);
  if (p->mode == MOE_MODE_AUTO && p->block_m != 0 && p->block_m != 16 && p->block_m != 32 && p->block_m != 64 &&
      p->block_m != 128)
    return fail(MOE_ERR_INVALID, "block_m %d not in {16, 32, 64, 128}", p->block_m);
  return MOE_OK;
}

// Tile orientation and block size.  Swap-AB when an expert is expected to see
// few tokens (the MMA M dimension is then filled by weight rows); the block
// is the smallest of 16/32/64 that usually holds an expert's tokens whole.
// The switch sits at 16 expected tokens per hit expert: there, with evenly
// spread routing, swap-AB tiles are a little faster, but with skewed routing
// the hot experts' many 16/32-row blocks each re-stream their weights and
// the 128-row tiles win by far more; the host cannot see the skew.
void resolve(moe_problem* p) {
  if (p->weight_dtype == MOE_DTYPE_MXFP8_E4M3) {  // block-scaled MMA: normal tiles only
    p->mode = MOE_MODE_NORMAL;
    p->block_m = 128;
    return;
  }
  // assignments expected on this call's experts (all of them without expert parallelism)
  const int64_t n = static_cast<int64_t>(p->T) * p->topk * p->E / global_experts(p);
  const int64_t hit = n < p->E ? n : p->E;
  const double avg = hit > 0 ? static_cast<double>(n) / static_cast<double>(hit) : 1.0;
  if (p->mode == MOE_MODE_AUTO) {
    if (p->block_m >= 128)
      p->mode = MOE_MODE_NORMAL;
    else if (p->block_m != 0 || p->H % 256)  // normal tiles need H % 256 == 0
      p->mode = MOE_MODE_SWAP_AB;
    else
      p->mode = avg < 16.0 ? MOE_MODE_SWAP_AB : MOE_MODE_NORMAL;
  }
  if (p->block_m == 0) {
    if (p->mode == MOE_MODE_NORMAL)
      p->block_m = 128;
    else
      p->block_m = avg <= 8.0 ? 16 : (avg <= 20.0 ? 32 : 64);
  }
}

int64_t capacity_of(int64_t T, int64_t topk, int64_t E, int64_t bm) {
  const int64_t n = T * topk;
  if (n == 0) return 0;
  const int64_t bound = n + (n < E ? n : E) * (bm - 1);
  return (bound + bm - 1) / bm * bm;
}

struct Plan {
  moe_problem p;
  moe_workspace_layout L;
  int64_t nflat;
  bool fp8;   // 8-bit weights and activations (block-128 or MX scales)
  bool mx;    // MXFP8: E8M0 scale factors per 32 elements
  bool tok_gather;  // swap-AB: GEMM1 gathers token rows (TMA gather4) from x or its per-token copy;
                    // normal tiles read a sorted copy a1 [capacity, H] (gather4 is too slow for 128-row tiles)
  bool ep;          // expert parallelism: some assignments go to other ranks' experts
  moe::ExpertRange er;
};

int make_plan(const moe_problem* in, Plan* plan) {
  int rc = validate_problem(in);
  if (rc != MOE_OK) return rc;
  plan->p = *in;
  resolve(&plan->p);
  const moe_problem& p = plan->p;
  plan->mx = p.weight_dtype == MOE_DTYPE_MXFP8_E4M3;
  plan->fp8 = p.weight_dtype == MOE_DTYPE_FP8_E4M3 || plan->mx;
  plan->tok_gather = p.mode == MOE_MODE_SWAP_AB;
  plan->ep = expert_parallel(&p);
  plan->er = moe::ExpertRange{p.first_expert, global_experts(&p)};
  plan->nflat = static_cast<int64_t>(p.T) * p.topk;
  const int64_t cap = capacity_of(p.T, p.topk, p.E, p.block_m);
  if (cap >= (int64_t(1) << 31)) return fail(MOE_ERR_INVALID, "padded row capacity overflows int32");
  const int64_t elem = plan->fp8 ? 1 : 2;
  const int64_t chunks = moe::align_chunks(plan->nflat);
  moe_workspace_layout& L = plan->L;
  int64_t off = 0;
  auto take = [&](int64_t bytes) {
    const int64_t o = off;
    off += align256(bytes);
    return o;
  };
  L.status = take(4);
  L.topk_ids = take(plan->nflat * 4);
  L.topk_weights = take(plan->nflat * 4);
  L.sorted_token_ids = take(cap * 4);
  L.expert_ids = take(cap / p.block_m * 4);
  L.num_tokens_post_padded = take(4);
  L.expert_counts = take(static_cast<int64_t>(p.E) * 4);
  L.expert_offsets = take(static_cast<int64_t>(p.E + 1) * 4);
  L.align_scratch = take(chunks * p.E * 4);
  // GEMM1's token rows: normal tiles read a sorted copy [cap, H]; swap-AB tiles
  // gather rows of x itself (bf16) or of its per-token copy [T, H] (quantised,
  // or scaled by the router weight)
  const bool rw = p.router_weight_on_input == 1;
  if (!plan->tok_gather)
    L.a1 = take(cap * p.H * elem);
  else if (plan->fp8 || rw)
    L.a1 = take(static_cast<int64_t>(p.T) * p.H * elem);
  else
    L.a1 = -1;
  // the inverse permutation: FP8 scale scatter, and the combine's mask under expert parallelism
  L.pos_of_flat = (plan->fp8 || plan->ep) ? take(plan->nflat * 4) : -1;
  // FP8: fp32 [K/128, cap]; MXFP8: E8M0 SF atoms, (cap/128) * (K/128) * 512 bytes -- the same size
  L.a1_scale = plan->fp8 ? take(cap * (p.H / 128) * 4) : -1;
  L.a2 = take(cap * p.I * elem);
  L.a2_scale = plan->fp8 ? take(cap * (p.I / 128) * 4) : -1;
  L.y = take(plan->nflat * p.H * 2);
  if (p.mode == MOE_MODE_SWAP_AB) {
    // one buffer serves both GEMMs (they run one after the other); GEMM1's
    // units hold 2*block_m accumulator columns, GEMM2's block_m
    L.partials = take(static_cast<int64_t>(moe::kMaxSplitUnits) * 128 * 2 * p.block_m * 4);
  } else {
    L.partials = -1;
  }
  L.total_bytes = off;
  L.capacity = static_cast<int32_t>(cap);
  L.block_m = p.block_m;
  L.mode = p.mode;
  L.align_chunks = static_cast<int32_t>(chunks);
  return MOE_OK;
}

template <typename T>
T* at(void* ws, int64_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

int run_stages(const moe_problem* prob, const void* x, const float* logits, const int32_t* topk_ids,
               const float* topk_weights, const void* w13, const void* w2, const void* w13_scale,
               const void* w2_scale, void* out, void* ws, size_t ws_bytes, int stage_begin, int stage_end,
               cudaStream_t stream) {
  Plan plan;
  int rc = make_plan(prob, &plan);
  if (rc != MOE_OK) return rc;
  const moe_problem& p = plan.p;
  const moe_workspace_layout& L = plan.L;
  if (stage_begin < 0 || stage_end > MOE_NUM_STAGES || stage_begin > stage_end)
    return fail(MOE_ERR_INVALID, "stage range [%d, %d)", stage_begin, stage_end);
  if (p.T == 0) return MOE_OK;  // nothing to read or write; buffers of zero rows may be NULL
  if (!x || !w13 || !w2 || !out || !ws) return fail(MOE_ERR_INVALID, "x, w13, w2, out and ws are required");
  if (!logits && (!topk_ids || !topk_weights))
    return fail(MOE_ERR_INVALID, "give router_logits, or topk_ids and topk_weights");
  if (plan.fp8 && (!w13_scale || !w2_scale)) return fail(MOE_ERR_INVALID, "FP8 weights need w13_scale and w2_scale");
  if (plan.mx && (!aligned(w13_scale, 16) || !aligned(w2_scale, 16)))
    return fail(MOE_ERR_INVALID, "MXFP8 scale factors must be 16-byte aligned");
  if (!aligned(x, 16) || !aligned(w13, 16) || !aligned(w2, 16) || !aligned(out, 16))
    return fail(MOE_ERR_INVALID, "x, w13, w2 and out must be 16-byte aligned");
  if ((logits && !aligned(logits, 4)) || (topk_ids && !aligned(topk_ids, 4)) ||
      (topk_weights && !aligned(topk_weights, 4)) || (w13_scale && !aligned(w13_scale, 4)) ||
      (w2_scale && !aligned(w2_scale, 4)))
    return fail(MOE_ERR_INVALID, "logits, routing and scale arrays must be 4-byte aligned");
  if (!aligned(ws, 256)) return fail(MOE_ERR_INVALID, "workspace must be 256-byte aligned");
  if (ws_bytes < static_cast<size_t>(L.total_bytes))
    return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes, need %lld", ws_bytes,
                static_cast<long long>(L.total_bytes));
  int sms = 0;
  rc = device_check(&sms);
  if (rc != MOE_OK) return rc;
  if (stage_begin == stage_end) return MOE_OK;

  int* status = at<int>(ws, L.status);
  const int32_t* ids = logits ? at<int32_t>(ws, L.topk_ids) : topk_ids;
  const float* wts = logits ? at<float>(ws, L.topk_weights) : topk_weights;
  const int nflat = static_cast<int>(plan.nflat);
  const int cap = L.capacity;
  const bool small = moe::route_align_small_fits(plan.nflat, plan.er.e_global);
  const bool swap = p.mode == MOE_MODE_SWAP_AB;
  int32_t* pos = L.pos_of_flat >= 0 ? at<int32_t>(ws, L.pos_of_flat) : nullptr;
  // GEMM1's token source: the sorted copy (normal tiles), the per-token copy, or x
  const void* tok_src = L.a1 >= 0 ? at<void>(ws, L.a1) : x;
  bool aligned_already = false;
  cudaError_t e;

  // the whole layer of a small bf16 batch in one persistent cooperative launch
  if (stage_begin == 0 && stage_end == MOE_NUM_STAGES && p.persistent_decode == 1 && !plan.fp8 && swap && !plan.ep &&
      p.block_m == moe::kDecodeBlockM && p.router_weight_on_input == 0 &&
      moe::decode_fused_fits(p.T, p.E, p.topk, p.H, p.I)) {
    int* sync = at<int>(ws, L.partials);  // the split-K buffer is not used by this path
    if ((e = cudaMemsetAsync(status, 0, sizeof(int), stream)) != cudaSuccess ||
        (e = cudaMemsetAsync(sync, 0, moe::kDecodeSyncInts * sizeof(int), stream)) != cudaSuccess)
      return cuda_fail(e, "clear sync words");
    moe::DecodeProblem dp{};
    dp.T = p.T;
    dp.E = p.E;
    dp.topk = p.topk;
    dp.H = p.H;
    dp.I = p.I;
    dp.renormalize = p.renormalize;
    dp.capacity = cap;
    dp.swiglu_limit = p.swiglu_limit > 0.0f ? p.swiglu_limit : INFINITY;
    dp.logits = logits;
    dp.ids_in = logits ? nullptr : topk_ids;
    dp.weights_in = logits ? nullptr : topk_weights;
    dp.x = x;
    dp.w13 = w13;
    dp.w2 = w2;
    dp.topk_ids = at<int32_t>(ws, L.topk_ids);
    dp.topk_weights = at<float>(ws, L.topk_weights);
    dp.sorted_ids = at<int32_t>(ws, L.sorted_token_ids);
    dp.expert_ids = at<int32_t>(ws, L.expert_ids);
    dp.ntpp = at<int32_t>(ws, L.num_tokens_post_padded);
    dp.counts = at<int32_t>(ws, L.expert_counts);
    dp.offsets = at<int32_t>(ws, L.expert_offsets);
    dp.a2 = at<void>(ws, L.a2);
    dp.y = at<void>(ws, L.y);
    dp.out = out;
    dp.sync = sync;
    dp.status = status;
    dp.num_sms = sms;
    e = moe::launch_decode_fused(dp, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "persistent decode");
  }

  for (int s = stage_begin; s < stage_end; ++s) {
    switch (s) {
      case MOE_STAGE_ROUTE:
        if ((e = cudaMemsetAsync(status, 0, sizeof(int), stream)) != cudaSuccess)
          return cuda_fail(e, "clear status");
        if (small && stage_end > MOE_STAGE_ALIGN) {
          // small batch: routing and the alignment in one single-CTA kernel
          e = moe::launch_route_align_small(logits, logits ? nullptr : topk_ids, p.T, p.E, plan.er, p.topk,
                                            p.renormalize, at<int32_t>(ws, L.topk_ids), at<float>(ws, L.topk_weights),
                                            p.block_m,
                                            cap, at<int32_t>(ws, L.sorted_token_ids), at<int32_t>(ws, L.expert_ids),
                                            at<int32_t>(ws, L.num_tokens_post_padded),
                                            at<int32_t>(ws, L.expert_counts), at<int32_t>(ws, L.expert_offsets),
                                            status, pos, stream);
          if (e != cudaSuccess) return cuda_fail(e, "route+align");
          aligned_already = true;
        } else if (logits) {
          e = moe::launch_route(logits, p.T, plan.er.e_global, p.topk, p.renormalize, at<int32_t>(ws, L.topk_ids),
                                at<float>(ws, L.topk_weights), stream);
          if (e != cudaSuccess) return cuda_fail(e, "route");
        }
        break;
      case MOE_STAGE_ALIGN:
        if (aligned_already) break;
        if (small) {
          e = moe::launch_route_align_small(nullptr, ids, p.T, p.E, plan.er, p.topk, p.renormalize, nullptr, nullptr,
                                            p.block_m, cap, at<int32_t>(ws, L.sorted_token_ids),
                                            at<int32_t>(ws, L.expert_ids), at<int32_t>(ws, L.num_tokens_post_padded),
                                            at<int32_t>(ws, L.expert_counts), at<int32_t>(ws, L.expert_offsets),
                                            status, pos, stream);
          if (e != cudaSuccess) return cuda_fail(e, "align");
          break;
        }
        e = moe::launch_align(ids, nflat, p.E, plan.er, p.block_m, cap, at<int32_t>(ws, L.sorted_token_ids),
                              at<int32_t>(ws, L.expert_ids), at<int32_t>(ws, L.num_tokens_post_padded),
                              at<int32_t>(ws, L.expert_counts), at<int32_t>(ws, L.expert_offsets),
                              at<int32_t>(ws, L.align_scratch), nullptr, nullptr, status, pos, stream);
        if (e != cudaSuccess) return cuda_fail(e, "align");
        break;
      case MOE_STAGE_GATHER:
        if (!plan.tok_gather && plan.fp8) {
          // normal FP8 / MXFP8 tiles: quantise once per token into the (not yet used)
          // y region, scattering the scales to the sorted rows, then copy code rows
          void* xq = at<void>(ws, L.y);
          e = moe::launch_prepare_x(x, p.T, p.H, p.topk, true, plan.mx, pos, cap,
                                    p.router_weight_on_input == 1 ? wts : nullptr, xq, at<void>(ws, L.a1_scale),
                                    stream);
          if (e == cudaSuccess)
            e = moe::launch_copy_rows(xq, p.H, p.topk, nflat, pos, at<void>(ws, L.a1), stream);
        } else if (!plan.tok_gather)
          e = moe::launch_gather(x, p.H, p.topk, nflat, at<int32_t>(ws, L.sorted_token_ids),
                                 at<int32_t>(ws, L.num_tokens_post_padded), cap, plan.fp8, plan.mx,
                                 p.router_weight_on_input == 1 ? wts : nullptr, at<void>(ws, L.a1),
                                 plan.fp8 ? at<void>(ws, L.a1_scale) : nullptr, stream);
        else
          e = moe::launch_prepare_x(x, p.T, p.H, p.topk, plan.fp8, plan.mx, pos, cap,
                                    p.router_weight_on_input == 1 ? wts : nullptr,
                                    L.a1 >= 0 ? at<void>(ws, L.a1) : nullptr,
                                    plan.fp8 ? at<void>(ws, L.a1_scale) : nullptr, stream);
        if (e != cudaSuccess) return cuda_fail(e, "gather");
        break;
      case MOE_STAGE_GEMM1:
      case MOE_STAGE_GEMM2: {
        moe::GemmProblem gp{};
        gp.E = p.E;
        gp.H = p.H;
        gp.I = p.I;
        gp.topk = p.topk;
        gp.nflat = nflat;
        gp.block_m = p.block_m;
        gp.capacity = cap;
        gp.fp8 = plan.fp8;
        gp.mx = plan.mx;
        gp.swap = swap;
        gp.ntpp = at<int32_t>(ws, L.num_tokens_post_padded);
        gp.expert_ids = at<int32_t>(ws, L.expert_ids);
        gp.sorted_ids = at<int32_t>(ws, L.sorted_token_ids);
        gp.topk_weights = wts;
        gp.status = status;
        gp.num_sms = sms;
        gp.split_mode = p.split_k;
        gp.partials = swap ? at<float>(ws, L.partials) : nullptr;
        gp.weight_on_input = p.router_weight_on_input == 1;
        gp.gather_tok = plan.tok_gather;
        gp.T = p.T;
        gp.swiglu_limit = p.swiglu_limit > 0.0f ? p.swiglu_limit : INFINITY;
        if (s == MOE_STAGE_GEMM1) {
          e = moe::launch_gemm1(gp, tok_src, plan.fp8 ? at<void>(ws, L.a1_scale) : nullptr, w13,
                                w13_scale, at<void>(ws, L.a2), plan.fp8 ? at<void>(ws, L.a2_scale) : nullptr,
                                stream);
          if (e != cudaSuccess) return cuda_fail(e, "gemm1");
        } else {
          e = moe::launch_gemm2(gp, at<void>(ws, L.a2), plan.fp8 ? at<void>(ws, L.a2_scale) : nullptr, w2,
                                w2_scale, at<void>(ws, L.y), stream);
          if (e != cudaSuccess) return cuda_fail(e, "gemm2");
        }
        break;
      }
      case MOE_STAGE_COMBINE:
        e = moe::launch_combine(at<void>(ws, L.y), p.T, p.topk, p.H, plan.ep ? pos : nullptr, out, stream);
        if (e != cudaSuccess) return cuda_fail(e, "combine");
        break;
      default:
        break;
    }
  }
  return MOE_OK;
}

int combine_allreduce(int32_t T, int32_t topk, int32_t H, int32_t world, int32_t rank, const moe_allreduce_rank* ranks,
                      uint32_t epoch, uint32_t timeout_us, void* stream, bool emulated, bool scatter) {
  if (world < 1 || world > MOE_MAX_RANKS) return fail(MOE_ERR_INVALID, "allreduce: world %d outside [1, %d]", world,
                                                      MOE_MAX_RANKS);
  if (!emulated && (rank < 0 || rank >= world)) return fail(MOE_ERR_INVALID, "allreduce: rank %d outside [0, %d)", rank,
                                                            world);
  if (T < 0 || topk < 1 || topk > 32 || H <= 0 || H % 128)
    return fail(MOE_ERR_INVALID, "allreduce: T=%d topk=%d H=%d (H a positive multiple of 128)", T, topk, H);
  if (static_cast<int64_t>(T) * topk * (scatter ? world : 1) >= (int64_t(1) << 31))
    return fail(MOE_ERR_INVALID, "allreduce: rows * topk overflows int32");
  if (epoch < 1 || epoch > 0x7FFFFFFFu) return fail(MOE_ERR_INVALID, "allreduce: epoch %u outside [1, 2^31)", epoch);
  if (timeout_us < 1 || timeout_us > 10000000u)
    return fail(MOE_ERR_INVALID, "allreduce: timeout_us %u outside [1, 10000000]", timeout_us);
  if (T == 0) return MOE_OK;
  if (!ranks) return fail(MOE_ERR_INVALID, "allreduce: ranks is NULL");
  moe::AllreduceRank r[moe::kMaxRanks] = {};
  for (int p = 0; p < world; ++p) {
    const moe_allreduce_rank& q = ranks[p];
    const bool own = emulated || p == rank;  // buffers this rank's kernel reads besides partial / out / flags
    if (!q.partial || !q.out || !q.flags || (own && (!q.y || !q.status)))
      return fail(MOE_ERR_INVALID, "allreduce: NULL buffer of rank %d", p);
    if (!aligned(q.partial, 16) || !aligned(q.out, 16) || !aligned(q.flags, 4) || (own && !aligned(q.y, 16)) ||
        (own && !aligned(q.pos_of_flat, 4)) || (own && !aligned(q.status, 4)))
      return fail(MOE_ERR_INVALID, "allreduce: misaligned buffer of rank %d", p);
    r[p] = moe::AllreduceRank{q.y, q.pos_of_flat, q.partial, q.out, q.flags, q.status};
  }
  int sms = 0;
  int rc = device_check(&sms);
  if (rc != MOE_OK) return rc;
  cudaError_t e = moe::launch_combine_allreduce(r, world, emulated ? -1 : rank, T, topk, H, scatter, epoch,
                                                1000ull * timeout_us, sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "allreduce");
}


}  // namespace

namespace moe {
int record_error(int code, const char* msg) { return fail(code, "%s", msg); }
}  // namespace moe

extern "C" {

const char* moe_last_error_string(void) { return g_last_error.c_str(); }

int32_t moe_version(void) { return 200; }

int moe_selftest_wait_timeout(uint32_t timeout_us, int32_t* status, uint64_t* waited_ns, void* stream) {
  if (timeout_us < 1 || timeout_us > 1000000)
    return fail(MOE_ERR_INVALID, "selftest: timeout_us %u outside [1, 1000000]", timeout_us);
  if (!status || !waited_ns) return fail(MOE_ERR_INVALID, "selftest: NULL pointer");
  if (!aligned(status, 4) || !aligned(waited_ns, 8)) return fail(MOE_ERR_INVALID, "selftest: misaligned pointer");
  int rc = device_check(nullptr);
  if (rc != MOE_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
  if (e == cudaSuccess)
    e = moe::launch_wait_selftest(reinterpret_cast<int*>(status), 1000ull * timeout_us,
                                  reinterpret_cast<unsigned long long*>(waited_ns), s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "selftest");
}

int moe_route(const float* logits, int32_t T, int32_t E, int32_t topk, int32_t renormalize, int32_t* topk_ids,
              float* topk_weights, void* stream) {
  if (T < 0 || E < 1 || E > 1024 || topk < 1 || topk > E || topk > 32)
    return fail(MOE_ERR_INVALID, "route: T=%d E=%d topk=%d (need T >= 0, 1 <= topk <= min(E, 32), E <= 1024)", T, E,
                topk);
  if (renormalize != 0 && renormalize != 1) return fail(MOE_ERR_INVALID, "route: renormalize must be 0 or 1");
  if (T > 0 && (!logits || !topk_ids || !topk_weights)) return fail(MOE_ERR_INVALID, "route: NULL pointer");
  if (!aligned(logits, 4) || !aligned(topk_ids, 4) || !aligned(topk_weights, 4))
    return fail(MOE_ERR_INVALID, "route: arrays must be 4-byte aligned");
  int rc = device_check(nullptr);
  if (rc != MOE_OK) return rc;
  cudaError_t e = moe::launch_route(logits, T, E, topk, renormalize, topk_ids, topk_weights,
                                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "route");
}

int64_t moe_align_capacity(int32_t T, int32_t topk, int32_t E, int32_t block_m) {
  if (T < 0 || topk < 1 || E < 1 || block_m < 1) return -1;
  return capacity_of(T, topk, E, block_m);
}

size_t moe_align_workspace_size(int32_t T, int32_t topk, int32_t E) {
  if (T < 0 || topk < 1 || E < 1) return 0;
  const int64_t n = static_cast<int64_t>(T) * topk;
  return static_cast<size_t>(align256(4) + align256(static_cast<int64_t>(E) * 4) + align256((E + 1) * 4LL) +
                             align256(static_cast<int64_t>(moe::align_chunks(n)) * E * 4));
}

int moe_align(const int32_t* topk_ids, int32_t T, int32_t topk, int32_t E, int32_t block_m, int32_t* sorted_token_ids,
              int32_t* expert_ids, int32_t* num_tokens_post_padded, int32_t* expert_counts, int32_t* expert_offsets,
              void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || topk < 1 || E < 1 || E > 1024 || block_m < 1 || block_m > 4096)
    return fail(MOE_ERR_INVALID, "align: T=%d topk=%d E=%d block_m=%d", T, topk, E, block_m);
  const int64_t n = static_cast<int64_t>(T) * topk;
  if (n >= (int64_t(1) << 31)) return fail(MOE_ERR_INVALID, "align: T * topk overflows int32");
  const int64_t cap = capacity_of(T, topk, E, block_m);
  if (cap >= (int64_t(1) << 31)) return fail(MOE_ERR_INVALID, "align: capacity overflows int32");
  if (!sorted_token_ids || !expert_ids || !num_tokens_post_padded || !ws || (n > 0 && !topk_ids))
    return fail(MOE_ERR_INVALID, "align: NULL pointer");
  if (!aligned(ws, 256)) return fail(MOE_ERR_INVALID, "align: workspace must be 256-byte aligned");
  if (ws_bytes < moe_align_workspace_size(T, topk, E))
    return fail(MOE_ERR_WORKSPACE, "align: workspace of %zu bytes, need %zu", ws_bytes,
                moe_align_workspace_size(T, topk, E));
  int rc = device_check(nullptr);
  if (rc != MOE_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(w);
  int32_t* counts = reinterpret_cast<int32_t*>(w + align256(4));
  int32_t* offs = reinterpret_cast<int32_t*>(w + align256(4) + align256(E * 4LL));
  int32_t* scratch = reinterpret_cast<int32_t*>(w + align256(4) + align256(E * 4LL) + align256((E + 1) * 4LL));
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e != cudaSuccess) return cuda_fail(e, "align: clear status");
  if (n == 0) {
    e = cudaMemsetAsync(num_tokens_post_padded, 0, sizeof(int32_t), s);
    if (e == cudaSuccess && expert_counts) e = cudaMemsetAsync(expert_counts, 0, E * sizeof(int32_t), s);
    if (e == cudaSuccess && expert_offsets) e = cudaMemsetAsync(expert_offsets, 0, (E + 1) * sizeof(int32_t), s);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "align");
  }
  if (moe::route_align_small_fits(n, E)) {
    e = moe::launch_route_align_small(nullptr, topk_ids, T, E, moe::ExpertRange{0, E}, topk, 1, nullptr, nullptr,
                                      block_m,
                                      static_cast<int>(cap), sorted_token_ids, expert_ids, num_tokens_post_padded,
                                      expert_counts ? expert_counts : counts, expert_offsets ? expert_offsets : offs,
                                      status, nullptr, s);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "align");
  }
  e = moe::launch_align(topk_ids, static_cast<int>(n), E, moe::ExpertRange{0, E}, block_m, static_cast<int>(cap),
                        sorted_token_ids,
                        expert_ids, num_tokens_post_padded, counts, offs, scratch, expert_counts, expert_offsets,
                        status, nullptr, s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "align");
}

int moe_quantize_weights_fp8(const void* w, int64_t batches, int32_t rows, int32_t cols, uint8_t* codes,
                             float* scales, void* stream) {
  if (batches < 0 || rows <= 0 || cols <= 0 || rows % 128 || cols % 128)
    return fail(MOE_ERR_INVALID, "quantize: batches=%lld rows=%d cols=%d (rows, cols multiples of 128)",
                static_cast<long long>(batches), rows, cols);
  if (batches > 0 && (!w || !codes || !scales)) return fail(MOE_ERR_INVALID, "quantize: NULL pointer");
  if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(scales, 4))
    return fail(MOE_ERR_INVALID, "quantize: w and codes 16-byte aligned, scales 4-byte aligned");
  int rc = device_check(nullptr);
  if (rc != MOE_OK) return rc;
  cudaError_t e = moe::launch_quantize_weights(w, batches, rows, cols, codes, scales, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "quantize");
}

int moe_quantize_weights_mxfp8(const void* w, int64_t batches, int32_t rows, int32_t cols, uint8_t* codes,
                               uint8_t* sf, void* stream) {
  if (batches < 0 || rows <= 0 || cols <= 0 || rows % 128 || cols % 128)
    return fail(MOE_ERR_INVALID, "quantize: batches=%lld rows=%d cols=%d (rows, cols multiples of 128)",
                static_cast<long long>(batches), rows, cols);
  if (batches > 0 && (!w || !codes || !sf)) return fail(MOE_ERR_INVALID, "quantize: NULL pointer");
  if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(sf, 16))
    return fail(MOE_ERR_INVALID, "quantize: w, codes and sf must be 16-byte aligned");
  int rc = device_check(nullptr);
  if (rc != MOE_OK) return rc;
  cudaError_t e = moe::launch_quantize_weights_mx(w, batches, rows, cols, codes, sf, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "quantize");
}

int32_t moe_combine_allreduce_flag_count(int32_t T, int32_t world) {
  if (T < 0 || world < 1 || world > MOE_MAX_RANKS) return 0;
  return 2 * moe::allreduce_chunks(T, world, false).nchunks + 1;
}

int32_t moe_combine_reduce_scatter_flag_count(int32_t T, int32_t world) {
  if (T < 0 || world < 1 || world > MOE_MAX_RANKS) return 0;
  return 2 * moe::allreduce_chunks(T, world, true).nchunks + 1;
}


int moe_combine_allreduce(int32_t T, int32_t topk, int32_t H, int32_t world, int32_t rank,
                          const moe_allreduce_rank* ranks, uint32_t epoch, uint32_t timeout_us, void* stream) {
  return combine_allreduce(T, topk, H, world, rank, ranks, epoch, timeout_us, stream, false, false);
}

int moe_combine_allreduce_emulated(int32_t T, int32_t topk, int32_t H, int32_t world, const moe_allreduce_rank* ranks,
                                   uint32_t epoch, uint32_t timeout_us, void* stream) {
  return combine_allreduce(T, topk, H, world, 0, ranks, epoch, timeout_us, stream, true, false);
}

int moe_combine_reduce_scatter(int32_t T, int32_t topk, int32_t H, int32_t world, int32_t rank,
                               const moe_allreduce_rank* ranks, uint32_t epoch, uint32_t timeout_us, void* stream) {
  return combine_allreduce(T, topk, H, world, rank, ranks, epoch, timeout_us, stream, false, true);
}

int moe_combine_reduce_scatter_emulated(int32_t T, int32_t topk, int32_t H, int32_t world,
                                        const moe_allreduce_rank* ranks, uint32_t epoch, uint32_t timeout_us,
                                        void* stream) {
  return combine_allreduce(T, topk, H, world, 0, ranks, epoch, timeout_us, stream, true, true);
}

int moe_resolve_problem(moe_problem* p) {
  int rc = validate_problem(p);
  if (rc != MOE_OK) return rc;
  resolve(p);
  return MOE_OK;
}

size_t moe_workspace_size(const moe_problem* p) {
  Plan plan;
  if (make_plan(p, &plan) != MOE_OK) return 0;
  return static_cast<size_t>(plan.L.total_bytes);
}

int moe_get_workspace_layout(const moe_problem* p, moe_workspace_layout* layout) {
  if (layout == nullptr) return fail(MOE_ERR_INVALID, "layout is NULL");
  Plan plan;
  int rc = make_plan(p, &plan);
  if (rc != MOE_OK) return rc;
  *layout = plan.L;
  return MOE_OK;
}

int moe_fused_forward(const moe_problem* p, const void* x, const float* router_logits, const int32_t* topk_ids,
                      const float* topk_weights, const void* w13, const void* w2, const void* w13_scale,
                      const void* w2_scale, void* out, void* ws, size_t ws_bytes, void* stream) {
  return run_stages(p, x, router_logits, topk_ids, topk_weights, w13, w2, w13_scale, w2_scale, out, ws, ws_bytes, 0,
                    MOE_NUM_STAGES, static_cast<cudaStream_t>(stream));
}

int moe_forward_stages(const moe_problem* p, const void* x, const float* router_logits, const int32_t* topk_ids,
                       const float* topk_weights, const void* w13, const void* w2, const void* w13_scale,
                       const void* w2_scale, void* out, void* ws, size_t ws_bytes, int32_t stage_begin,
                       int32_t stage_end, void* stream) {
  return run_stages(p, x, router_logits, topk_ids, topk_weights, w13, w2, w13_scale, w2_scale, out, ws, ws_bytes,
                    stage_begin, stage_end, static_cast<cudaStream_t>(stream));
}

int moe_read_status(const moe_problem* p, void* ws, int32_t clear, int32_t* status, void* stream) {
  if (!ws || !status) return fail(MOE_ERR_INVALID, "read_status: NULL pointer");
  Plan plan;
  int rc = make_plan(p, &plan);
  if (rc != MOE_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* dev = at<int>(ws, plan.L.status);
  cudaError_t e = cudaMemcpyAsync(status, dev, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(dev, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "read_status");
}

}  // extern "C"
