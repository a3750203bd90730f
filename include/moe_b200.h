/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) fused top-k Mixture-of-Experts layer.
 *
 * The layer computes, for every token t of x[T, H]:
 *
 *   route   : topk_ids[t, :], topk_weights[t, :] from router logits (softmax
 *             over E experts, the k largest, renormalised), or given;
 *   align   : the flat assignments t*topk + j sorted by expert and padded to
 *             whole blocks of block_m rows (sorted_token_ids, expert_ids);
 *   GEMM1   : h = x[t] . w13[e]^T  (w13[e] is [2I, H]; gate = rows [0, I),
 *             up = rows [I, 2I)), held in bf16;
 *   act     : a2 = bf16(bf16(silu(gate)) * up), re-quantised to FP8 E4M3 per
 *             (row, 128 columns) with a power-of-two scale on the FP8 path;
 *   GEMM2   : y[t*topk + j] = topk_weights[t, j] * (a2 . w2[e]^T)  (w2[e] is [H, I]);
 *   combine : out[t] = sum_j y[t*topk + j].
 *
 * Sources: "AWS erklärt zwei Kernel-Optimierungen, die den Durchsatz von
 * SageMaker AI auf H200 steigern" (kinachrichten.com), sections "Warum
 * MoE-Kernel so wichtig sind" (fused routing + expert compute) and "Swap-AB"
 * (weight rows fill the MMA M dimension at decode); the analysis of vLLM PR
 * #64760 "FP8 MoE down-projection for H200" (blog.secrett2633.cloud), §1.1
 * (expert-sorted intermediate, sorted_token_ids / num_tokens_post_padded,
 * block-padded rows) and §1.2 (fused SiLU-mul-FP8 quantisation kernel); and
 * "Hosting von Qwen auf Blackwell" (perplexity.ai), section "MoE Dispatch -
 * Combine" (weighted accumulation in the combine).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned and allocated by the
 *    caller, row-major and contiguous.  The library allocates no device or
 *    host memory on these paths and keeps no per-call state.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *    is asynchronous on it: it enqueues kernels and returns.  No call
 *    synchronises the device unless its comment says so.
 *  - Return value: MOE_OK, or a negative MOE_ERR_* code; on error
 *    moe_last_error_string() (per host thread) describes it.  Arguments are
 *    validated before anything is enqueued, so an error return means nothing
 *    was launched (MOE_ERR_CUDA excepted: a launch failed part way).
 *  - Bad device data (an expert id outside [0, E), or outside
 *    [0, num_global_experts) under expert parallelism) cannot be seen on the
 *    host: the kernels record it in the workspace status word (see
 *    moe_read_status) and the outputs of that call are undefined.
 */
#ifndef MOE_B200_H_
#define MOE_B200_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define MOE_OK 0
#define MOE_ERR_INVALID (-1)     /* null pointer, bad shape, misaligned pointer */
#define MOE_ERR_UNSUPPORTED (-2) /* not an sm_100 device, unsupported combination */
#define MOE_ERR_WORKSPACE (-3)   /* workspace smaller than moe_workspace_size() */
#define MOE_ERR_CUDA (-4)        /* a CUDA call or kernel launch failed */

/* device status word codes (moe_read_status) */
#define MOE_STATUS_OK 0
#define MOE_STATUS_BAD_EXPERT_ID 1    /* an expert id outside [0, E) (num_global_experts under EP) */
#define MOE_STATUS_WAIT_TIMEOUT 0x100 /* a bounded in-kernel wait ran out; low byte = where */

/* weight types */
#define MOE_DTYPE_BF16 0
#define MOE_DTYPE_FP8_E4M3 1 /* E4M3 codes + one fp32 scale per 128 x 128 block */
#define MOE_DTYPE_MXFP8_E4M3 2 /* E4M3 codes + one E8M0 (power-of-two) scale per 32 elements of a row;
                                 normal tiles only (mode NORMAL, block_m 128) */

/*
 * MXFP8 scale-factor layout ("SF atoms"), used for MXFP8 weights and for the
 * activation scales the library writes.  For a matrix [.., N, K] (K the
 * reduction axis) the E8M0 byte of element (n, k) of batch b lives at
 *   ((b * (N/128) + n/128) * (K/128) + k/128) * 512
 *     + (n % 32) * 16 + ((n % 128) / 32) * 4 + (k % 128) / 32,
 * i.e. one contiguous 512-byte atom per 128 rows x 128 columns, in the order
 * the tensor cores read scale factors (tcgen05.cp 32x128b, 4 warps).  E8M0
 * byte v encodes 2^(v - 127).
 */

/* tile orientation of the two grouped GEMMs */
#define MOE_MODE_AUTO 0    /* swap-AB below 16 expected tokens per hit expert (T*topk/E), else normal */
#define MOE_MODE_NORMAL 1  /* MMA M = 128 token rows (block_m 128), N = 256 weight rows */
#define MOE_MODE_SWAP_AB 2 /* MMA M = 128 weight rows, N = block_m token rows */

/* stages of moe_forward_stages, in pipeline order */
#define MOE_STAGE_ROUTE 0   /* router (skipped without logits); for T*topk <= 8192 and E <= 256 it also aligns */
#define MOE_STAGE_ALIGN 1   /* histogram, scan, stable scatter (no work when the route stage aligned) */
#define MOE_STAGE_GATHER 2  /* x rows into expert-sorted order (+ FP8 quantisation) */
#define MOE_STAGE_GEMM1 3   /* gate/up grouped GEMM + fused SiLU*up (+ FP8 requant) */
#define MOE_STAGE_GEMM2 4   /* down grouped GEMM + routed-weight scatter */
#define MOE_STAGE_COMBINE 5 /* per-token sum of its topk rows */
#define MOE_NUM_STAGES 6

/*
 * Problem description.  T, E, topk, H, I and weight_dtype are required;
 * mode = MOE_MODE_AUTO and block_m = 0 let the library choose; both are
 * written back by moe_resolve_problem().
 * Constraints: T >= 0, 1 <= topk <= E <= 1024 (topk <= num_global_experts
 * under expert parallelism, below), H and I positive multiples of
 * 128, T * topk < 2^31.  Normal tiles (and so MXFP8) cover 256 columns of H
 * per GEMM2 tile and need H % 256 == 0; MOE_MODE_AUTO picks swap-AB tiles
 * when H % 256 == 128.
 */
typedef struct moe_problem {
  int32_t T;            /* tokens */
  int32_t E;            /* experts */
  int32_t topk;         /* experts per token */
  int32_t H;            /* hidden size */
  int32_t I;            /* expert intermediate size */
  int32_t weight_dtype; /* MOE_DTYPE_* */
  int32_t mode;         /* MOE_MODE_* */
  int32_t block_m;      /* rows per expert block: 16, 32, 64 (swap-AB); 128 (normal); 0 = auto */
  int32_t renormalize;  /* router: 1 = renormalise the chosen softmax weights (default), 0 = keep them */
  int32_t split_k;      /* swap-AB GEMMs: 0 = split K when few tiles are in flight (default), 1 = never */
  /* 1 = scale each token row by its router weight before GEMM1 instead of the
   * expert output after GEMM2 (vLLM's apply_router_weight_on_input, shown
   * False in the PR analysis' test); requires topk == 1.  0 = default. */
  int32_t router_weight_on_input;
  /* SwiGLU clamp limit L > 0: gate = min(gate, L), up = clamp(up, -L, L) before
   * SiLU(gate) * up (the clamp_limit that the PR analysis' sorted-A predicate
   * excludes).  0 = no clamp (default). */
  float swiglu_limit;
  /* moe_fused_forward of a small bf16 batch (T * topk <= 256, E <= 256, swap-AB
   * block_m 16, weights on the output): 1 = the whole layer in one persistent
   * cooperative launch, 0 = the kernel-per-stage pipeline (default: measured
   * faster, the persistent kernel is opt-in). */
  int32_t persistent_decode;
  /* Expert parallelism ("Hosting von Qwen auf Blackwell", section "MoE
   * Dispatch - Combine", "Experten-Parallel": x and the routing are the same
   * on every rank; each rank runs only the assignments to its own experts,
   * sums them per token, and an all-reduce over the ranks completes the
   * layer).  The router scores num_global_experts experts (router_logits is
   * [T, num_global_experts]; topk_ids hold global ids in
   * [0, num_global_experts)), while this call holds the weights of the E
   * experts [first_expert, first_expert + E) only: w13 [E, 2I, H] and
   * w2 [E, H, I] are those experts' weights, local expert e is global expert
   * first_expert + e, and expert_counts / expert_offsets / expert_ids in the
   * workspace are local.  Assignments to other experts are skipped (not an
   * error), so out[t] is the sum over t's local assignments only, zero when
   * it has none; the sum of out over a partition of the experts is the
   * layer.  Constraints: E <= num_global_experts <= 1024, 0 <= first_expert
   * <= num_global_experts - E, topk <= num_global_experts.  0 and 0 = every
   * expert is local (num_global_experts = E). */
  int32_t num_global_experts;
  int32_t first_expert;
  int32_t reserved[1];  /* must be zero */
} moe_problem;

/*
 * Byte offsets of the intermediates inside the workspace (for inspection
 * by tests and tools; all regions are 256-byte aligned).  A region a call
 * does not use has offset -1.
 */
typedef struct moe_workspace_layout {
  int64_t status;           /* int32 status word */
  int64_t topk_ids;         /* int32 [T*topk]      (router output) */
  int64_t topk_weights;     /* fp32  [T*topk]      (router output) */
  int64_t sorted_token_ids; /* int32 [capacity] */
  int64_t expert_ids;       /* int32 [capacity / block_m] */
  int64_t num_tokens_post_padded; /* int32 */
  int64_t expert_counts;    /* int32 [E] (local experts under expert parallelism) */
  int64_t expert_offsets;   /* int32 [E + 1] */
  int64_t align_scratch;    /* int32 [chunks * E] */
  int64_t pos_of_flat;      /* int32 [T*topk]: sorted row of each assignment, -1 for a bad id or another
                               rank's expert (FP8 / MXFP8, and every expert-parallel call) */
  int64_t a1;               /* GEMM1 token rows.  Normal tiles: x rows in sorted order [capacity, H], bf16 or
                               E4M3 (padding rows unspecified).  Swap-AB: one row per token [T, H] -- E4M3
                               codes (FP8) or bf16(x * w) (router weight on the input) -- gathered by TMA;
                               -1 when GEMM1 gathers straight from x */
  int64_t a1_scale;         /* fp32 [H/128, capacity] (FP8, K-block major); E8M0 SF atoms of [capacity, H] (MXFP8) */
  int64_t a2;               /* bf16 or E4M3 [capacity, I] activation in sorted order (padding rows unspecified) */
  int64_t a2_scale;         /* fp32 [I/128, capacity] (FP8, K-block major); E8M0 SF atoms of [capacity, I] (MXFP8) */
  int64_t y;                /* bf16 [T*topk, H] weighted expert outputs (rows of other ranks' assignments
                               unwritten under expert parallelism) */
  int64_t partials;         /* fp32 split-K partial sums of the swap-AB GEMMs (swap-AB only) */
  int64_t total_bytes;
  int32_t capacity;         /* rows of sorted_token_ids */
  int32_t block_m;
  int32_t mode;
  int32_t align_chunks;
} moe_workspace_layout;

/* Human-readable description of the last error on this host thread. */
MOE_API const char* moe_last_error_string(void);

/*
 * Top-k softmax router ("Warum MoE-Kernel so wichtig sind": token routing).
 * logits [T, E] fp32 -> topk_ids [T, topk] int32, topk_weights [T, topk] fp32.
 * Experts are taken by descending logit, equal logits by the lower index;
 * weights are softmax probabilities (renormalize = 0) or those renormalised
 * over the chosen experts (renormalize = 1).  One warp per token.
 */
MOE_API int moe_route(const float* logits, int32_t T, int32_t E, int32_t topk, int32_t renormalize,
              int32_t* topk_ids, float* topk_weights, void* stream);

/*
 * Rows of sorted_token_ids for a problem: an upper bound of
 * sum_e ceil(count_e / block_m) * block_m, namely
 * block_m * ceil((T*topk + min(E, T*topk) * (block_m - 1)) / block_m).
 * Returns -1 on invalid arguments.
 */
MOE_API int64_t moe_align_capacity(int32_t T, int32_t topk, int32_t E, int32_t block_m);

/* Scratch bytes moe_align() needs (per-chunk expert histograms). */
MOE_API size_t moe_align_workspace_size(int32_t T, int32_t topk, int32_t E);

/*
 * Expert alignment (vLLM PR #64760 analysis, §1.1: sorted_token_ids,
 * num_tokens_post_padded, one expert per BLOCK_SIZE_M rows).
 *   topk_ids [T, topk] int32 in [0, E).
 *   sorted_token_ids [capacity] int32: the flat ids t*topk + j of expert 0,
 *     then expert 1, ..., each expert's run in ascending flat order and padded
 *     with the sentinel T*topk to a multiple of block_m; the sentinel also
 *     fills [num_tokens_post_padded, capacity).
 *   expert_ids [capacity / block_m] int32: the expert of each used block, -1 after.
 *   num_tokens_post_padded [1] int32.
 *   expert_counts [E], expert_offsets [E + 1] int32: may be NULL.
 *   ws / ws_bytes: scratch of at least moe_align_workspace_size() bytes.
 * Deterministic: the result is a pure function of topk_ids.
 */
MOE_API int moe_align(const int32_t* topk_ids, int32_t T, int32_t topk, int32_t E, int32_t block_m,
              int32_t* sorted_token_ids, int32_t* expert_ids, int32_t* num_tokens_post_padded,
              int32_t* expert_counts, int32_t* expert_offsets, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_align without a workspace, for callers that cannot allocate device
 * memory when they align (a framework that owns every allocation and lends
 * none, code running inside a CUDA-graph capture with a fixed memory plan,
 * a serving loop that bans allocator calls after start-up).  The pages have
 * no counterpart of this entry point; it is a deployment convenience.
 *
 * Same arguments, results and determinism as moe_align, minus ws/ws_bytes:
 * the scratch moe_align would take from the workspace lives instead in one
 * static device array of MOE_ALIGN_NOALLOC_SCRATCH_BYTES, which every GPU
 * that loads this library holds until the process exits.
 *  - Limit: moe_align_workspace_size(T, topk, E) must not exceed
 *    MOE_ALIGN_NOALLOC_SCRATCH_BYTES (1 MiB: about 520 000 assignments at
 *    E = 128, 260 000 at E = 256); larger problems return MOE_ERR_INVALID
 *    before anything is enqueued.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.  The address is kept for the life of the
 *    process: after cudaDeviceReset on a device, do not call this entry point
 *    on that device again.  A failed lookup returns MOE_ERR_CUDA with the CUDA
 *    error's name and text in moe_last_error_string().
 *  - All calls on a device share the array, and it keeps the previous
 *    call's contents; each call clears or rewrites every entry it reads.
 *    Calls whose executions overlap on the GPU (unordered streams) race.
 *  - An expert id outside [0, E) is not reported (the status word lives in
 *    the shared array); the outputs of that call are then undefined.
 *  - Calls no allocator (no cudaMalloc, cudaFree or allocating library call).
 */
#define MOE_ALIGN_NOALLOC_SCRATCH_BYTES (1 << 20)
MOE_API int moe_align_noalloc(const int32_t* topk_ids, int32_t T, int32_t topk, int32_t E, int32_t block_m,
                              int32_t* sorted_token_ids, int32_t* expert_ids, int32_t* num_tokens_post_padded,
                              int32_t* expert_counts, int32_t* expert_offsets, void* stream);

/*
 * FP8 weight preparation: w [batches, rows, cols] bf16 -> codes [batches,
 * rows, cols] E4M3 and scales [batches, rows/128, cols/128] fp32 with, per
 * 128 x 128 block, scale = max(blockmax, 1e-10) / 448 (fp32) and
 * code = e4m3(fp32(w / scale)) (round to nearest even, saturating).
 * rows and cols must be multiples of 128.
 */
MOE_API int moe_quantize_weights_fp8(const void* w, int64_t batches, int32_t rows, int32_t cols, uint8_t* codes,
                             float* scales, void* stream);

/*
 * MXFP8 weight preparation ("Hosting von Qwen auf Blackwell", section
 * "Quantisierung": micro-scaled FP8 weights on Blackwell).  w [batches, rows,
 * cols] bf16 -> codes [batches, rows, cols] E4M3 and E8M0 scale factors in the
 * SF-atom layout above (batches * rows * cols / 32 bytes).  Per row and 32
 * consecutive columns: scale = the smallest power of two >= fp32(max(amax,
 * 1e-10)) * fp32(1/448), code = e4m3(w / scale) (exact division, round to
 * nearest even, saturating).  rows and cols must be multiples of 128; codes
 * 16-byte and sf 16-byte aligned.
 */
MOE_API int moe_quantize_weights_mxfp8(const void* w, int64_t batches, int32_t rows, int32_t cols, uint8_t* codes,
                                       uint8_t* sf, void* stream);

/* Fill in mode and block_m when they are left to the library; validates p. */
MOE_API int moe_resolve_problem(moe_problem* p);

/* Workspace bytes moe_fused_forward needs for p (0 on invalid p). */
MOE_API size_t moe_workspace_size(const moe_problem* p);

/* Where each intermediate lives inside the workspace for p. */
MOE_API int moe_get_workspace_layout(const moe_problem* p, moe_workspace_layout* layout);

/*
 * The fused MoE layer, all stages on `stream`.
 *   x             [T, H] bf16.
 *   router_logits [T, E] fp32 ([T, num_global_experts] under expert
 *                 parallelism), or NULL to use topk_ids / topk_weights
 *                 ([T, topk] int32 / fp32, global expert ids), which are then required.
 *   w13           [E, 2I, H]: bf16, or E4M3 codes with w13_scale [E, 2I/128, H/128] fp32
 *                 (MOE_DTYPE_FP8_E4M3), or E4M3 codes with w13_scale as E8M0 SF atoms
 *                 of [E, 2I, H] (MOE_DTYPE_MXFP8_E4M3; x and the intermediate are then
 *                 MX-quantised the same way, per row and 32 columns).
 *   w2            [E, H, I]:  likewise, w2_scale [E, H/128, I/128] fp32 or SF atoms of [E, H, I].
 *   out           [T, H] bf16 (under expert parallelism: this rank's partial sum).
 *   ws            device scratch of at least moe_workspace_size(p) bytes,
 *                 256-byte aligned; the call clears what must start at zero.
 *                 Two calls that overlap on the device must not share it.
 * All pointers 16-byte aligned.  T = 0 is a no-op (its buffers may be NULL).
 */
MOE_API int moe_fused_forward(const moe_problem* p, const void* x, const float* router_logits, const int32_t* topk_ids,
                      const float* topk_weights, const void* w13, const void* w2, const void* w13_scale,
                      const void* w2_scale, void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * The same pipeline restricted to stages [stage_begin, stage_end) (MOE_STAGE_*),
 * so that a caller can time or inspect each stage.  Running every range of a
 * partition in order is exactly moe_fused_forward.
 */
MOE_API int moe_forward_stages(const moe_problem* p, const void* x, const float* router_logits, const int32_t* topk_ids,
                       const float* topk_weights, const void* w13, const void* w2, const void* w13_scale,
                       const void* w2_scale, void* out, void* ws, size_t ws_bytes, int32_t stage_begin,
                       int32_t stage_end, void* stream);

/*
 * Read (and with clear != 0, reset) the device status word of a workspace.
 * SYNCHRONISES `stream`.  Writes MOE_STATUS_* into *status.
 */
MOE_API int moe_read_status(const moe_problem* p, void* ws, int32_t clear, int32_t* status, void* stream);

/*
 * Failure-detection self-test (no counterpart on the pages).  Launches one
 * kernel whose only wait -- on an mbarrier nothing arrives at -- goes through
 * the same bounded wait the pipeline kernels use, limited to timeout_us
 * (1 .. 1 000 000).  It must give up: *status (device int32, cleared first)
 * receives MOE_STATUS_WAIT_TIMEOUT | 0x7F and *waited_ns (device uint64) the
 * time it waited; the kernel then returns normally and the context stays
 * usable.  Nothing faults, traps or hangs.
 */
MOE_API int moe_selftest_wait_timeout(uint32_t timeout_us, int32_t* status, uint64_t* waited_ns, void* stream);

/*
 * Fused combine + all-reduce of an expert-parallel layer ("Hosting von Qwen
 * auf Blackwell", section "MoE Dispatch - Combine", "Experten-Parallel": the
 * local accumulation, then an all-reduce over the ranks; section
 * "All-Reduce": the reduction split over the ranks, each reducing a part and
 * sending it to the others).  It replaces the combine stage of every rank's
 * moe_forward_stages(..., MOE_STAGE_ROUTE, MOE_STAGE_COMBINE, ...) call and
 * the all-reduce after it: one kernel per rank, over peer memory, in which
 * every token chunk is first summed locally (partial), then reduced by the
 * rank that owns the chunk (chunk c: rank c % world) from every rank's partial
 * in rank order (fp32, one bf16 rounding) and stored into every rank's out.
 *
 * moe_allreduce_rank: one rank's buffers, as mapped in the calling process
 * (peers' through CUDA peer mappings; all ranks on one NVLink domain).
 *   y, pos_of_flat  that rank's workspace regions "y" and "pos_of_flat"
 *                   (moe_get_workspace_layout of its expert-parallel problem);
 *                   read by that rank only.  pos_of_flat may be NULL when
 *                   every assignment has a row on the rank (a problem without
 *                   expert parallelism, whose layout may have no such region).
 *   partial, out    bf16 [T, H] each, 16-byte aligned; partial is read and out
 *                   written by every rank.
 *   flags           int32 [moe_combine_allreduce_flag_count(T, world)], zeroed
 *                   once by the caller before the first call; the same flags
 *                   serve every later call of the same T and world.
 *   status          int32 status word of the rank (e.g. its workspace's).
 * epoch: 1 for the first call on a set of flags, then one more per call (the
 * flags remember the last epoch; nothing is reset between calls).  Every rank
 * passes the same epoch, T, topk, H and world.
 * timeout_us (1 .. 10 000 000): every wait on another rank is bounded; one
 * that runs out records MOE_STATUS_WAIT_TIMEOUT | 0x31 (chunk ready) or 0x32
 * (chunk done) in the rank's status word, the rank's later waits of that call
 * give up at once, and the kernel returns (out is then incomplete).
 * Buffers of rows [0, T) only; T = 0 is a no-op.
 */
#define MOE_MAX_RANKS 16

typedef struct moe_allreduce_rank {
  const void* y;
  const int32_t* pos_of_flat;
  void* partial;
  void* out;
  int32_t* flags;
  int32_t* status;
} moe_allreduce_rank;

/* int32 entries of each rank's flags array for T tokens over world ranks (0 on bad arguments). */
MOE_API int32_t moe_combine_allreduce_flag_count(int32_t T, int32_t world);

/*
 * This rank's kernel (ranks[0 .. world) as mapped here, `rank` = the caller's
 * index).  Every rank must launch it for the same epoch; each returns when
 * its own out is complete.  The y, pos_of_flat and status of the other ranks
 * are not read and may be NULL.
 */
MOE_API int moe_combine_allreduce(int32_t T, int32_t topk, int32_t H, int32_t world, int32_t rank,
                                  const moe_allreduce_rank* ranks, uint32_t epoch, uint32_t timeout_us,
                                  void* stream);

/*
 * Every rank's kernel as one cooperative launch on the current device, with
 * all ranks' buffers in this device's memory: the same device code and the
 * same flag protocol, for testing the exchange on one GPU.
 */
MOE_API int moe_combine_allreduce_emulated(int32_t T, int32_t topk, int32_t H, int32_t world,
                                           const moe_allreduce_rank* ranks, uint32_t epoch, uint32_t timeout_us,
                                           void* stream);

/*
 * Reduce-scatter form, for data parallelism combined with expert parallelism
 * (the page's decoders: each rank serves its own requests while the experts
 * are sharded).  Every rank brings T tokens; the ranks' x and routing inputs
 * are gathered (rank r's tokens are rows [r*T, (r+1)*T) of the gathered
 * batch), every rank runs its expert share on the whole gathered batch of
 * world * T tokens, and this kernel then leaves in each rank's out [T, H] the
 * layer for that rank's own tokens: partial is [world * T, H], y and
 * pos_of_flat are those of the share's world*T-token problem, out is [T, H],
 * flags has moe_combine_reduce_scatter_flag_count(T, world) entries.  Rank r
 * reduces its own rows from every rank's partial (rank order, fp32, one bf16
 * rounding) and stores only into its own out.  Epochs, time limits, status
 * codes and the emulated form are as for the all-reduce above.
 */
MOE_API int32_t moe_combine_reduce_scatter_flag_count(int32_t T, int32_t world);
MOE_API int moe_combine_reduce_scatter(int32_t T, int32_t topk, int32_t H, int32_t world, int32_t rank,
                                       const moe_allreduce_rank* ranks, uint32_t epoch, uint32_t timeout_us,
                                       void* stream);
MOE_API int moe_combine_reduce_scatter_emulated(int32_t T, int32_t topk, int32_t H, int32_t world,
                                                const moe_allreduce_rank* ranks, uint32_t epoch,
                                                uint32_t timeout_us, void* stream);

/* Library version: major * 10000 + minor * 100 + patch. */
MOE_API int32_t moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H_ */
