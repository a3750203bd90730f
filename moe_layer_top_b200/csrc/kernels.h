// Host-side launchers of the MoE kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

namespace moe {

// Launch `kern` on `stream` with programmatic stream serialisation, so that
// it may start while the previous kernel of the stream finishes (each kernel
// calls griddepcontrol.wait before it reads what its predecessors wrote).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// router ---------------------------------------------------------------------
cudaError_t launch_route(const float* logits, int T, int E, int topk, int renormalize, int32_t* ids,
                         float* weights, cudaStream_t stream);

// align ----------------------------------------------------------------------
constexpr int kAlignChunk = 256;  // assignments per warp-chunk
inline int align_chunks(long long n) { return static_cast<int>((n + kAlignChunk - 1) / kAlignChunk); }

// Expert ranges (both align paths): the ids are global, in [0, e_global);
// local expert e is global expert first + e for e in [0, E).  Assignments to
// other experts are skipped silently; ids outside [0, e_global) are reported.
// Without expert parallelism first = 0 and e_global = E.
struct ExpertRange {
  int first;
  int e_global;
};

cudaError_t launch_align(const int32_t* topk_ids, int n, int E, ExpertRange er, int block_m, int capacity,
                         int32_t* sorted_ids, int32_t* expert_ids, int32_t* ntpp, int32_t* counts_ws,
                         int32_t* offsets_ws, int32_t* chunk_scratch, int32_t* user_counts,
                         int32_t* user_offsets, int* status, int32_t* pos_of_flat, cudaStream_t stream);

// single-CTA route (optional, over er.e_global experts) + align for small batches
constexpr int kSmallAlignMaxN = 8192;  // assignments (T * topk)
constexpr int kSmallAlignMaxE = 256;   // router width (e_global)
bool route_align_small_fits(long long n, int e_global);
cudaError_t launch_route_align_small(const float* logits, const int32_t* ids_in, int T, int E, ExpertRange er,
                                     int topk, int renormalize, int32_t* ids_out, float* weights_out, int block_m,
                                     int capacity, int32_t* sorted_ids, int32_t* expert_ids, int32_t* ntpp,
                                     int32_t* counts, int32_t* offsets, int* status, int32_t* pos_of_flat,
                                     cudaStream_t stream);

// pos_of_flat (optional, both align paths): sorted position of every flat
// assignment, -1 for an invalid or non-local expert id (the inverse of
// sorted_token_ids)

// gather x rows into sorted order: bf16 copy, FP8 per-(row,128) quantisation
// (a1_scale: fp32 [H/128, capacity]) or MXFP8 per-(row,32) quantisation
// (a1_scale: E8M0 SF atoms of [capacity, H])
// (row_weight != NULL: each row is first scaled by row_weight[flat], rounded to bf16)
cudaError_t launch_gather(const void* x, int H, int topk, int nflat, const int32_t* sorted_ids,
                          const int32_t* ntpp, int capacity, bool fp8, bool mx, const float* row_weight, void* a1,
                          void* a1_scale, cudaStream_t stream);

// x once per token, for GEMM1's TMA gather of token rows: FP8 / MXFP8 codes
// into xq [T, H] with each (token, K block) scale scattered to the sorted rows
// of its assignments (fp32 [H/128, capacity] or E8M0 SF atoms of [capacity, H]);
// bf16 with a router weight on the input: xq = bf16(x * w) [T, H]; plain bf16:
// nothing (GEMM1 reads x itself)
cudaError_t launch_prepare_x(const void* x, int T, int H, int topk, bool fp8, bool mx, const int32_t* pos_of_flat,
                             int capacity, const float* row_weight, void* xq, void* scales, cudaStream_t stream);

// a1[pos_of_flat[f]] = xq[f / topk] (E4M3 rows [T, H] -> sorted [capacity, H]) for every row-owning f
cudaError_t launch_copy_rows(const void* xq, int H, int topk, int nflat, const int32_t* pos_of_flat, void* a1,
                             cudaStream_t stream);

// out[t] = sum_j y[t*topk + j]; with pos_of_flat, only the assignments that
// have a row (pos_of_flat >= 0: local experts under expert parallelism)
cudaError_t launch_combine(const void* y, int T, int topk, int H, const int32_t* pos_of_flat, void* out,
                           cudaStream_t stream);

// FP8 128x128 block weight quantisation
cudaError_t launch_quantize_weights(const void* w, long long batches, int rows, int cols, uint8_t* codes,
                                    float* scales, cudaStream_t stream);

// MXFP8 weight quantisation: per (row, 32 columns) E8M0 scale, SF-atom layout
cudaError_t launch_quantize_weights_mx(const void* w, long long batches, int rows, int cols, uint8_t* codes,
                                       uint8_t* sf, cudaStream_t stream);

// grouped GEMMs ----------------------------------------------------------------
struct GemmProblem {
  int E, H, I, topk, nflat, block_m, capacity;
  bool fp8, swap;
  bool mx;             // MXFP8 (with fp8): block-scaled MMA, E8M0 SF atoms
  bool weight_on_input;  // the router weight was applied in the gather: GEMM2 stores y unweighted
  bool gather_tok;     // GEMM1: token rows come from a [T, H] source by sorted_ids / topk (TMA gather)
  int T;               // rows of that source
  float swiglu_limit;  // SwiGLU clamp limit (+inf: none)
  const int32_t* ntpp;
  const int32_t* expert_ids;
  const int32_t* sorted_ids;
  const float* topk_weights;  // [nflat]
  int* status;
  int num_sms;
  int split_mode;      // swap-AB split-K: 0 when few tiles are in flight, 1 never
  float* partials;     // swap-AB split-K partial sums [unit][acc column][128] (reused by both GEMMs)
};

// swap-AB split-K: at most this many (tile, split) units per launch
constexpr int kMaxSplitUnits = 320;  // >= 4 splits x (148 SMs / 2) tiles

// GEMM1 + fused SiLU*up (+ FP8 requant): a1 [cap, H] -> a2 [cap, I] (+ a2_scale_t [I/128, cap]).
// In swap-AB mode with split-K allowed this launches the GEMM and then the
// split-K reduce kernel (which exits at once when the GEMM did not split).
// Scale arguments: FP8 -- fp32 (activation scales K-block major, weight scales
// per 128x128 block); MXFP8 -- E8M0 SF atoms.
cudaError_t launch_gemm1(const GemmProblem& p, const void* a1, const void* a1_scale, const void* w13,
                         const void* w13_scale, void* a2, void* a2_scale, cudaStream_t stream);

// GEMM2 + routed weight: a2 [cap, I] -> y [nflat, H] bf16 (rows scattered by sorted_ids);
// swap-AB split-K launches the reduce kernel after it, as for GEMM1
cudaError_t launch_gemm2(const GemmProblem& p, const void* a2, const void* a2_scale, const void* w2,
                         const void* w2_scale, void* y, cudaStream_t stream);

// 2-D K-major TMA tensor map: [rows, cols] elements of elem_bytes, box = 128
// bytes x box_rows, 128-byte swizzle (box_rows = 1 for tile::gather4 maps)
bool make_tma_map_2d(CUtensorMap* map, const void* base, long long rows, long long cols, int elem_bytes,
                     int box_rows);

// persistent decode kernel (route + align + GEMM1 + GEMM2 + combine in one
// cooperative launch) for small bf16 batches; see decode_fused.cu
struct DecodeProblem {
  int T, E, topk, H, I, renormalize, capacity;
  float swiglu_limit;  // +inf: none
  const float* logits;             // [T, E] or NULL
  const int32_t* ids_in;           // [T, topk] when logits == NULL
  const float* weights_in;         // [T, topk] when logits == NULL
  const void* x;                   // [T, H] bf16
  const void* w13;                 // [E, 2I, H] bf16
  const void* w2;                  // [E, H, I] bf16
  int32_t* topk_ids;               // router output [T, topk]
  float* topk_weights;             // router output [T, topk]
  int32_t* sorted_ids;             // [capacity]
  int32_t* expert_ids;             // [capacity / 16]
  int32_t* ntpp;
  int32_t* counts;                 // [E]
  int32_t* offsets;                // [E + 1]
  void* a2;                        // [capacity, I] bf16
  void* y;                         // [T * topk, H] bf16
  void* out;                       // [T, H] bf16
  int* sync;                       // kDecodeSyncInts ints, zeroed before the launch
  int* status;
  int num_sms;
};
constexpr int kDecodeMaxAssignments = 256;   // T * topk
constexpr int kDecodeMaxExperts = 256;
constexpr int kDecodeBlockM = 16;
constexpr int kDecodeSyncInts = 8 + kDecodeMaxAssignments + kDecodeMaxExperts;  // flags + ready[block]
bool decode_fused_fits(int T, int E, int topk, int H, int I);
cudaError_t launch_decode_fused(const DecodeProblem& p, cudaStream_t stream);

// failure-detection self-test: one bounded wait that must time out
cudaError_t launch_wait_selftest(int* status, unsigned long long timeout_ns, unsigned long long* waited_ns,
                                 cudaStream_t stream);

// set the per-thread error message returned by moe_last_error_string(); returns code
int record_error(int code, const char* msg);

// shared-memory bytes the GEMM variant needs (for validation / occupancy)
size_t gemm_smem_bytes(bool gemm2, bool fp8, bool swap, int block_m);

}  // namespace moe
