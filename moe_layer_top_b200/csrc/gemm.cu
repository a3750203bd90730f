// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// GEMM1 (gate/up):  h[r, :] = x(r) . w13[e(r)]^T, followed in the epilogue
//   by a2 = bf16(bf16(silu(gate)) * up) and, on the FP8 path, the per-(row,128)
//   power-of-two E4M3 re-quantisation (vLLM PR #64760 analysis, §1.2: the
//   fused SiLU-mul-quant kernel, here fused into the GEMM epilogue so the bf16
//   intermediate never reaches HBM).
// GEMM2 (down):     y[flat(r), :] = topk_weight(flat(r)) * a2[r, :] . w2[e(r)]^T,
//   reading a2 in expert-sorted order with plain TMA tiles (§1.1, sorted-A)
//   and scattering rows to their flat assignment index.
//
// Rows are the expert-sorted, block-padded assignments produced by align; a
// block of block_m rows belongs to one expert.  Two tile orientations:
//   normal : MMA M = 128 token rows, N = 256 weight rows (GEMM1: 128 gate +
//            128 up rows of one 128-column intermediate group);
//   swap-AB: MMA M = 128 weight rows, N = block_m token rows -- the
//            orientation the AWS/kinachrichten page ("Swap-AB") describes for
//            decode batches, where the token count cannot fill the MMA M.
//
// Kernel structure (one CTA per SM, persistent over tiles, 10 warps):
//   warp 0     : TMA producer (one lane issues; for swap-AB GEMM1 the whole
//                warp first stages the tile's token row ids, which the lane
//                then gathers with tile::gather4 from x or its per-token FP8
//                copy), multi-stage smem ring;
//   warp 1     : TMEM allocator and MMA issuer (one lane);
//   warps 2..9 : epilogue, two groups of four warps (each group covers the
//                128 TMEM lanes; the groups split the accumulator columns).
// bf16: the whole K reduction accumulates in TMEM (double-buffered across
// tiles).  FP8: weights carry one fp32 scale per 128x128 block and activations
// one power-of-two scale per (row, 128); every 128-deep K block accumulates
// into its own TMEM buffer (double-buffered) and the epilogue promotes it into
// fp32 registers with the product of the two scales.  MXFP8 (separate kernel
// below): E8M0 scales per 32 elements applied inside block-scaled MMAs.
// Launch chain: GEMM1 lets GEMM2 launch only after its own dependency wait,
// so GEMM2 streams its first weight stages before waiting on GEMM1.  Swap-AB
// problems with at most half as many tiles as SMs split K; a reduce kernel
// adds the splits.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;
constexpr int kSmemLimit = 232448;  // max dynamic shared memory per block on sm_100
constexpr int kSmemReserve = 4096;  // barriers, TMEM slot, exchange buffers
constexpr int kXchgOffset = 512;    // exchange buffers (2 x 256 floats) start here
constexpr int kTokRowsOffset = 3072; // token row ids of the current tile (<= 128 int32) for the TMA gather

// wait-site codes reported in the status word (low byte)
constexpr int kWhereProducer = 1, kWhereMma = 2, kWhereEpiAcc = 3, kWhereEpiXchg = 4, kWhereDrain = 5;

constexpr int ceil_pow2(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

template <bool kDown, bool kFP8, bool kSwap, int kBM>
struct Cfg {
  static constexpr int kKElems = kFP8 ? 128 : 64;  // K elements per stage (128 bytes per row)
  static constexpr int kTokRows = kSwap ? kBM : 128;
  static constexpr int kWRows = (kSwap && kDown) ? 128 : 256;
  static constexpr int kTokBytes = kTokRows * 128;
  static constexpr int kWBytes = kWRows * 128;
  static constexpr int kStageBytes = kTokBytes + kWBytes;
  // GEMM2 FP8 normal tiles stage each output row in shared memory and write it with one
  // asynchronous bulk copy (256 contiguous bytes per row): a thread's own row stored from
  // registers would take 16 scattered 16-byte stores, which cost a third of the kernel.  The
  // staging area (pitch 272 bytes: 16-byte aligned, 4-way bank spread) takes one ring stage.
  // GEMM1 FP8 normal tiles do the same with their 64-byte FP8 row chunks (four scattered 16-byte stores).
  static constexpr bool kStageY = kFP8 && !kSwap;
  static constexpr int kYPitch = kDown ? 272 : 80;
  static constexpr int kYStageBytes = kStageY ? 256 * kYPitch : 0;
  static constexpr int kStagesFit = (kSmemLimit - kSmemReserve - 1024 - kYStageBytes) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kMmaN = kSwap ? kBM : 256;
  static constexpr int kAccCols = kSwap ? (kDown ? kBM : 2 * kBM) : 256;
  // TMEM accumulator buffers.  bf16: two (the whole K range of a tile accumulates in one; the
  // next tile's MMAs use the other).  FP8: one per 128-deep K block; swap-AB accumulators are
  // narrow, so up to eight let the MMA run that many K blocks ahead of the epilogue's
  // promotion (a normal tile's 256 columns leave room for two).
  static constexpr int kAccBufs = kFP8 ? ((512 / kAccCols) > 8 ? 8 : (512 / kAccCols)) : 2;
  static constexpr int kTmemCols = ceil_pow2((kAccBufs * kAccCols) < 32 ? 32 : kAccBufs * kAccCols);
  // output columns per tile: GEMM1 -> 128 intermediate columns; GEMM2 -> H columns
  static constexpr int kTileN = kDown ? (kSwap ? 128 : 256) : 128;
  static constexpr int kHalfTok = kBM / 2;  // swap: token columns per epilogue group
  static constexpr size_t kSmemBytes =
      static_cast<size_t>(kStages) * kStageBytes + kSmemReserve + kYStageBytes + 1024;
  static_assert(kStages >= 2, "pipeline needs at least two stages");
  static_assert(kSmemBytes <= static_cast<size_t>(kSmemLimit), "shared memory");
  static_assert(kTmemCols <= 512, "TMEM holds 512 columns");
  static_assert(kAccBufs >= 2, "accumulators are at least double-buffered");
  static_assert((2 * kStages + 2 * kAccBufs + 3) * 8 + 8 <= kXchgOffset, "barriers overlap the exchange buffers");
  static_assert(!kSwap || kBM == 16 || kBM == 32 || kBM == 64, "swap-AB block_m");
};

struct Args {
  int E, H, I, nflat, capacity;
  const int32_t* ntpp;
  const int32_t* expert_ids;
  const int32_t* sorted_ids;
  const float* topk_weights;
  const float* a_scale_t;  // [K/128, capacity]
  const float* w_scale;    // [E, Nw/128, K/128]
  void* out;               // GEMM1: a2 [capacity, I]; GEMM2: y [nflat, H]
  float* out_scale_t;      // GEMM1 FP8: a2 scale [I/128, capacity]
  int* status;
  float* partials;         // swap-AB split-K: [unit][acc column][128] fp32 partial sums
  int splits;              // swap-AB split-K factor S (1: no split); chosen on the host
  float swiglu_limit;      // GEMM1: SwiGLU clamp limit (+inf: none)
  int gather_tok;          // GEMM1: token rows are gathered from the [T, K] source by sorted_ids / topk
  int topk;
  const uint8_t* a_sf;     // MXFP8: E8M0 SF atoms of the activation rows [capacity, K]
  const uint8_t* w_sf;     // MXFP8: E8M0 SF atoms of the weights [E * Nw, K]
  uint8_t* out_sf;         // MXFP8 GEMM1: SF atoms of a2 [capacity, I]
};

// Split-K for the swap-AB tiles: when at most half the SMs would have a tile
// (few experts hit and small H or I), the K range of every tile is cut in S
// pieces so that more SMs stream weights.  Each split stores fp32 partial
// sums; a reduce kernel adds them in split order (deterministic) and runs the
// epilogue.  S is chosen on the host from the tile count bound that the
// capacity gives (capacity / block_m blocks), so the host knows whether the
// reduce kernel is needed.  A split needs >= 4 K stages, and a launch at most
// kMaxSplitUnits units (the partial-sum buffer).
constexpr int kMaxSplits = 4;

int choose_splits(long long tiles, int ctas, int k_stages) {
  if (tiles <= 0 || 2 * tiles > ctas) return 1;
  int best = 1;
  long long best_u = tiles, best_w = (tiles + ctas - 1) / ctas;  // efficiency = u / (ctas * w)
  for (int sp = 2; sp <= kMaxSplits; ++sp) {
    if (k_stages / sp < 4 || tiles * sp > kMaxSplitUnits) break;
    const long long u = tiles * sp, w = (u + ctas - 1) / ctas;
    if (u * best_w * 100 > best_u * w * 105) {  // at least 5 % better
      best = sp;
      best_u = u;
      best_w = w;
    }
  }
  return best;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status,
                                          int where) {
  const bool ok = mbar_wait(bar, parity, abort, status, MOE_STATUS_WAIT_TIMEOUT | where);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void store_bf16x16(__nv_bfloat16* dst, const float (&v)[16]) {
  uint4 u[2];
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(u);
#pragma unroll
  for (int i = 0; i < 8; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  reinterpret_cast<uint4*>(dst)[0] = u[0];
  reinterpret_cast<uint4*>(dst)[1] = u[1];
}

template <bool kDown, bool kFP8, bool kSwap, int kBM>
__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tm_tok, const __grid_constant__ CUtensorMap tm_w,
                    const Args args) {
  using C = Cfg<kDown, kFP8, kSwap, kBM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* reserve = smem + static_cast<size_t>(C::kStages) * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(reserve);
  uint64_t* empty = full + C::kStages;
  uint64_t* acc_full = empty + C::kStages;
  uint64_t* acc_empty = acc_full + C::kAccBufs;
  uint64_t* xchg_bar = acc_empty + C::kAccBufs;
  uint64_t* drain = xchg_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xchg = reinterpret_cast<float*>(reserve + kXchgOffset);  // [2][2 * 128] floats

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if constexpr (kDown) pdl_launch_dependents();  // GEMM1 triggers only after its own wait (below)
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    for (int b = 0; b < 2; ++b) mbar_init(&xchg_bar[b], kEpiWarps * 32);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_tok);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // GEMM1 waits here, then lets GEMM2 launch: GEMM2 may then read the alignment
  // (written two or more launches back) before its own wait and start streaming
  // its weights under GEMM1's tail.  GEMM2 waits per role.
  if constexpr (!kDown) {
    pdl_wait();
    pdl_launch_dependents();
  }

  const int H = args.H, I = args.I;
  const int K = kDown ? I : H;                           // reduction length
  const int rows_per_block = C::kTokRows;                // == block_m of the alignment
  const int n_tiles = (kDown ? H : I) / C::kTileN;
  const int num_mblocks = (kDown ? ld_cg_i32(args.ntpp) : (*(args.ntpp))) / rows_per_block;
  const int num_tiles = num_mblocks * n_tiles;
  const int k_stages = K / C::kKElems;
  const int splits = kSwap ? args.splits : 1;
  const int num_units = num_tiles * splits;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if constexpr (kDown) {
      // GEMM2: the weight tiles of the first kStages fills are issued before the
      // wait (they depend only on the alignment); the a2 tiles follow after it.
      if (lane == 0) {
        // weights: read once per expert by swap-AB tiles (evict first), but by every 128-row block of
        // the expert in the normal orientation, whose blocks run in the same wave (keep in L2)
        const uint64_t pol_w = kSwap ? policy_evict_first() : policy_evict_normal();
        const uint64_t pol_a = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        long long fills = 0;
        bool ok = true;
        int unit = static_cast<int>(blockIdx.x) - static_cast<int>(gridDim.x);
        int ks = 0, ks_end = 0, tok_row = 0, w_row = 0;
        auto advance = [&]() -> bool {  // next (unit, K stage) of this CTA
          if (ks + 1 < ks_end) {
            ++ks;
            return true;
          }
          unit += static_cast<int>(gridDim.x);
          if (unit >= num_units) return false;
          const int tile = unit / splits, split = unit - tile * splits;
          ks = split * k_stages / splits;
          ks_end = (split + 1) * k_stages / splits;
          const int mb = tile / n_tiles, nt = tile - mb * n_tiles;
          tok_row = mb * rows_per_block;
          w_row = ld_cg_i32(args.expert_ids + mb) * H + nt * C::kTileN;
          return ks < ks_end;
        };
        int pre_kx[C::kStages], pre_row[C::kStages];
        int npre = 0;
        bool more = true;
        while (npre < C::kStages && (more = advance())) {
          uint8_t* st = smem + static_cast<size_t>(stage) * C::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          const int kx = ks * C::kKElems;
          tma_load_2d(st + C::kTokBytes, &tm_w, &full[stage], kx, w_row, pol_w);
          pre_kx[npre] = kx;
          pre_row[npre] = tok_row;
          ++npre;
          ++fills;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        pdl_wait();  // a2 (GEMM1's output) is complete from here on
        for (int i = 0; i < npre; ++i)
          tma_load_2d(smem + static_cast<size_t>(i) * C::kStageBytes, &tm_tok, &full[i], pre_kx[i], pre_row[i],
                      pol_a);
        while (more && ok && (more = advance())) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, args.status,
                         MOE_STATUS_WAIT_TIMEOUT | kWhereProducer)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + static_cast<size_t>(stage) * C::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          const int kx = ks * C::kKElems;
          tma_load_2d(st, &tm_tok, &full[stage], kx, tok_row, pol_a);
          tma_load_2d(st + C::kTokBytes, &tm_w, &full[stage], kx, w_row, pol_w);
          ++fills;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) {
          for (int s = 0; s < C::kStages; ++s) {
            const long long n_s = fills / C::kStages + (s < fills % C::kStages ? 1 : 0);
            if (n_s > 0) {
              const uint64_t t0 = globaltimer_ns();
              while (!mbar_try_wait(&full[s], static_cast<uint32_t>((n_s - 1) & 1)) &&
                     globaltimer_ns() - t0 < kWaitTimeoutNs) {
              }
            }
          }
        }
      }
    } else {
    // All 32 lanes stage the tile's token row ids (GEMM1 gathers token rows
    // from x or its quantised copy); lane 0 issues every TMA load.
    int32_t* tok_rows = reinterpret_cast<int32_t*>(reserve + kTokRowsOffset);
    // weights: read once per expert by swap-AB tiles (evict first), but by every 128-row block of
    // the expert in the normal orientation, whose blocks run in the same wave (keep in L2)
    const uint64_t pol_w = kSwap ? policy_evict_first() : policy_evict_normal();
    const uint64_t pol_a = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    long long fills = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < num_units && ok; unit += gridDim.x) {
      const int tile = unit / splits, split = unit - tile * splits;
      const int ks0 = split * k_stages / splits, ks1 = (split + 1) * k_stages / splits;
      const int mb = tile / n_tiles, nt = tile - mb * n_tiles;
      const int tok_row = mb * rows_per_block;
      if (args.gather_tok) {
        for (int i = lane; i < C::kTokRows; i += 32) {
          const int f = (*(args.sorted_ids + tok_row + i));
          tok_rows[i] = f < args.nflat ? f / args.topk : 0;  // padding rows read any valid row
        }
      }
      __syncwarp();
      if (lane == 0) {
        const int e = (*(args.expert_ids + mb));
        int w_row0, w_row1;
        if constexpr (kDown) {
          w_row0 = e * H + nt * C::kTileN;
          w_row1 = w_row0;
        } else {
          w_row0 = e * 2 * I + nt * 128;      // gate rows
          w_row1 = w_row0 + I;                // up rows
        }
        for (int ks = ks0; ks < ks1; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, args.status,
                         MOE_STATUS_WAIT_TIMEOUT | kWhereProducer)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + static_cast<size_t>(stage) * C::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          const int kx = ks * C::kKElems;
          if (args.gather_tok) {
#pragma unroll 4
            for (int g = 0; g < C::kTokRows / 4; ++g) {
              const int4 r4 = reinterpret_cast<const int4*>(tok_rows)[g];
              tma_gather4(st + 512 * g, &tm_tok, &full[stage], kx, r4.x, r4.y, r4.z, r4.w);
            }
          } else {
            tma_load_2d(st, &tm_tok, &full[stage], kx, tok_row, pol_a);
          }
          if constexpr (kDown) {
            tma_load_2d(st + C::kTokBytes, &tm_w, &full[stage], kx, w_row0, pol_w);
          } else {
            tma_load_2d(st + C::kTokBytes, &tm_w, &full[stage], kx, w_row0, pol_w);
            tma_load_2d(st + C::kTokBytes + 16384, &tm_w, &full[stage], kx, w_row1, pol_w);
          }
          ++fills;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      __syncwarp();  // the row ids are rewritten only after lane 0 issued this tile's loads
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0 && !ok) {
      // let every copy already issued land before the CTA tears down
      for (int s = 0; s < C::kStages; ++s) {
        const long long n_s = fills / C::kStages + (s < fills % C::kStages ? 1 : 0);
        if (n_s > 0) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[s], static_cast<uint32_t>((n_s - 1) & 1)) &&
                 globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
    }  // GEMM1 producer
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if constexpr (kDown) pdl_wait();
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(128, C::kMmaN, kFP8);
      int stage = 0, abuf = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < num_units && ok; unit += gridDim.x) {
        const int split = unit % splits;
        const int ks0 = split * k_stages / splits, ks1 = (split + 1) * k_stages / splits;
        if constexpr (!kFP8) {
          if (!mbar_wait(&acc_empty[abuf], aphase ^ 1u, abort_flag, args.status,
                         MOE_STATUS_WAIT_TIMEOUT | kWhereMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        for (int ks = ks0; ks < ks1; ++ks) {
          if (!mbar_wait(&full[stage], phase, abort_flag, args.status, MOE_STATUS_WAIT_TIMEOUT | kWhereMma)) {
            ok = false;
            break;
          }
          if constexpr (kFP8) {
            if (!mbar_wait(&acc_empty[abuf], aphase ^ 1u, abort_flag, args.status,
                           MOE_STATUS_WAIT_TIMEOUT | kWhereMma)) {
              ok = false;
              break;
            }
          }
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(abuf * C::kAccCols);
          const uint32_t tok = smem_u32(smem + static_cast<size_t>(stage) * C::kStageBytes);
          const uint32_t w = tok + C::kTokBytes;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t koff = k * 32;  // 16 bf16 or 32 e4m3 elements
            const uint32_t acc = kFP8 ? (k > 0 ? 1u : 0u) : ((ks > ks0 || k > 0) ? 1u : 0u);
            if constexpr (!kSwap) {
              const uint64_t ad = smem_desc_sw128(tok + koff), bd = smem_desc_sw128(w + koff);
              if constexpr (kFP8) mma_fp8(d, ad, bd, idesc, acc); else mma_bf16(d, ad, bd, idesc, acc);
            } else if constexpr (!kDown) {
              const uint64_t bd = smem_desc_sw128(tok + koff);
              const uint64_t ag = smem_desc_sw128(w + koff), au = smem_desc_sw128(w + 16384 + koff);
              if constexpr (kFP8) {
                mma_fp8(d, ag, bd, idesc, acc);
                mma_fp8(d + kBM, au, bd, idesc, acc);
              } else {
                mma_bf16(d, ag, bd, idesc, acc);
                mma_bf16(d + kBM, au, bd, idesc, acc);
              }
            } else {
              const uint64_t ad = smem_desc_sw128(w + koff), bd = smem_desc_sw128(tok + koff);
              if constexpr (kFP8) mma_fp8(d, ad, bd, idesc, acc); else mma_bf16(d, ad, bd, idesc, acc);
            }
          }
          mma_commit(&empty[stage]);
          if constexpr (kFP8) {
            mma_commit(&acc_full[abuf]);
            if (++abuf == C::kAccBufs) {
              abuf = 0;
              aphase ^= 1u;
            }
          }
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if constexpr (!kFP8) {
          mma_commit(&acc_full[abuf]);
          if (++abuf == C::kAccBufs) {
            abuf = 0;
            aphase ^= 1u;
          }
        }
      }
      // every MMA this thread issued has completed once `drain` flips
      // (waited on even after an abort: TMEM must not be freed under a running MMA)
      mma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0)) {
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
          report_status(args.status, MOE_STATUS_WAIT_TIMEOUT | kWhereDrain);
          break;
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    if constexpr (kDown) pdl_wait();
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int g = (warp - 2) >> 2;          // epilogue group
    const int row = 32 * q + lane;          // accumulator row (TMEM lane)
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    int abuf = 0;
    uint32_t aphase = 0;
    int xbuf = 0;
    uint32_t xphase = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < num_units && ok; unit += gridDim.x) {
      const int tile = unit / splits, split = unit - tile * splits;
      const int ks0 = split * k_stages / splits, ks1 = (split + 1) * k_stages / splits;
      const int mb = tile / n_tiles, nt = tile - mb * n_tiles;
      const int e = (*(args.expert_ids + mb));

      if constexpr (!kSwap) {
        // ---------------- normal: row = token row of the tile
        const int grow = mb * 128 + row;  // sorted row
        constexpr int kCols = kDown ? 128 : 64;  // accumulator columns per group (per gate/up half for GEMM1)
        // GEMM2: the row's flat assignment and routed weight, read before the K loop so that
        // their two dependent global loads are not on the tile's tail
        int flat = 0;
        float wt = 0.f;
        if constexpr (kDown) {
          flat = (*(args.sorted_ids + grow));
          wt = flat < args.nflat ? route_weight(args.topk_weights, flat) : 0.f;
        }
        float acc_a[kFP8 ? kCols : 1];
        float acc_b[(kFP8 && !kDown) ? kCols : 1];
        if constexpr (kFP8) {
#pragma unroll
          for (int i = 0; i < kCols; ++i) acc_a[i] = 0.f;
          if constexpr (!kDown) {
#pragma unroll
            for (int i = 0; i < kCols; ++i) acc_b[i] = 0.f;
          }
          const int kb_n = K / 128;
          const float* sa_p = args.a_scale_t + grow;
          const float* sw_a;
          const float* sw_b;
          if constexpr (kDown) {
            sw_a = args.w_scale + (static_cast<size_t>(e) * (H / 128) + nt * 2 + g) * kb_n;
            sw_b = sw_a;
          } else {
            sw_a = args.w_scale + (static_cast<size_t>(e) * (2 * I / 128) + nt) * kb_n;
            sw_b = args.w_scale + (static_cast<size_t>(e) * (2 * I / 128) + I / 128 + nt) * kb_n;
          }
          // the scales of K block kb are loaded two blocks ahead: their global-load latency
          // would otherwise sit between two accumulator drains on the MMA's critical path
          float sa0 = (*(sa_p)), swa0 = (*(sw_a)), swb0 = (*(sw_b));
          float sa1 = 0.f, swa1 = 0.f, swb1 = 0.f;
          if (kb_n > 1) {
            sa1 = (*(sa_p + static_cast<size_t>(args.capacity)));
            swa1 = (*(sw_a + 1));
            swb1 = (*(sw_b + 1));
          }
          for (int kb = 0; kb < kb_n; ++kb) {
            const float fa = sa0 * swa0;
            const float fb = sa0 * swb0;
            sa0 = sa1;
            swa0 = swa1;
            swb0 = swb1;
            if (kb + 2 < kb_n) {
              sa1 = (*(sa_p + static_cast<size_t>(kb + 2) * args.capacity));
              swa1 = (*(sw_a + kb + 2));
              swb1 = (*(sw_b + kb + 2));
            }
            if (!warp_wait(&acc_full[abuf], aphase, abort_flag, args.status, kWhereEpiAcc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t t0 = tmem_base + lane_addr + static_cast<uint32_t>(abuf * C::kAccCols);
            // Promotion, software-pipelined: chunk c+1 is loaded from TMEM while chunk c is
            // scaled into the fp32 accumulators (two lanes per instruction), and the buffer is
            // handed back to the MMA as soon as its last chunk has landed in registers.
            // (tcgen05.wait::ld waits for every load issued so far, so each wait comes before
            // the next chunk's load is issued.)
            constexpr int kChunks = kDown ? kCols / 16 : kCols / 8;
            constexpr int kW = kDown ? 16 : 8;                   // words per chunk (per gate/up half)
            uint32_t ba[2][kW], bb[2][kDown ? 1 : kW];
            auto load = [&](int c) {
              if constexpr (kDown) {
                tmem_ld16u(t0 + g * 128 + 16 * c, ba[c & 1]);
              } else {
                tmem_ld8u(t0 + g * 64 + 8 * c, ba[c & 1]);
                tmem_ld8u(t0 + 128 + g * 64 + 8 * c, bb[c & 1]);
              }
            };
            load(0);
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
              tmem_wait_ld();                                    // chunk c is in registers
              if (c + 1 < kChunks) {
                load(c + 1);                                     // in flight while chunk c is scaled
              } else {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[abuf]);    // the MMA may reuse the buffer
              }
#pragma unroll
              for (int i = 0; i < kW; i += 2) {
                ffma2f(acc_a[kW * c + i], acc_a[kW * c + i + 1], ba[c & 1][i], ba[c & 1][i + 1], fa);
                if constexpr (!kDown)
                  ffma2f(acc_b[kW * c + i], acc_b[kW * c + i + 1], bb[c & 1][i], bb[c & 1][i + 1], fb);
              }
            }
            if (++abuf == C::kAccBufs) {
              abuf = 0;
              aphase ^= 1u;
            }
          }
          if (!ok) break;
        }

        if constexpr (!kDown) {
          // ---- GEMM1 epilogue: SiLU(gate) * up, bf16 store or FP8 requant
          __nv_bfloat16* a2 = static_cast<__nv_bfloat16*>(args.out);
          const int col0 = nt * 128 + g * 64;  // intermediate column of this group's first value
          if constexpr (!kFP8) {
            if (!warp_wait(&acc_full[abuf], aphase, abort_flag, args.status, kWhereEpiAcc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t t0 = tmem_base + lane_addr + static_cast<uint32_t>(abuf * C::kAccCols);
            uint32_t packed[32];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float dg[16], du[16];
              tmem_ld16(t0 + g * 64 + 16 * c, dg);
              tmem_ld16(t0 + 128 + g * 64 + 16 * c, du);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float p0 = swiglu_bf16(bf16_round(dg[2 * i]), bf16_round(du[2 * i]), args.swiglu_limit);
                const float p1 =
                    swiglu_bf16(bf16_round(dg[2 * i + 1]), bf16_round(du[2 * i + 1]), args.swiglu_limit);
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                packed[8 * c + i] = *reinterpret_cast<const uint32_t*>(&h2);
              }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[abuf]);
            if (++abuf == C::kAccBufs) {
              abuf = 0;
              aphase ^= 1u;
            }
            uint4* dst = reinterpret_cast<uint4*>(a2 + static_cast<size_t>(grow) * I + col0);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          } else {
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const float p = swiglu_bf16(bf16_round(acc_a[i]), bf16_round(acc_b[i]), args.swiglu_limit);
              acc_a[i] = p;
              amax = fmaxf(amax, fabsf(p));
            }
            // the 128-column group spans both epilogue groups: exchange the row maxima
            float* xb = xchg + xbuf * 256;
            xb[g * 128 + row] = amax;
            mbar_arrive(&xchg_bar[xbuf]);
            if (!warp_wait(&xchg_bar[xbuf], xphase, abort_flag, args.status, kWhereEpiXchg)) {
              ok = false;
              break;
            }
            amax = fmaxf(xb[row], xb[128 + row]);
            xbuf ^= 1;
            if (xbuf == 0) xphase ^= 1u;
            const float scale = act_scale_from_amax(amax);
            const float inv = pow2_recip(scale);
            uint32_t words[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              words[i] = static_cast<uint32_t>(f32x2_to_e4m3x2(acc_a[4 * i] * inv, acc_a[4 * i + 1] * inv)) |
                         (static_cast<uint32_t>(f32x2_to_e4m3x2(acc_a[4 * i + 2] * inv, acc_a[4 * i + 3] * inv))
                          << 16);
            }
            // the row's 64 codes go out through shared memory as one bulk copy
            uint8_t* st_row = reserve + kSmemReserve + static_cast<size_t>(threadIdx.x - 64) * C::kYPitch;
            bulk_wait_read_all();   // the previous copy from this staging slot has read it
#pragma unroll
            for (int i = 0; i < 4; ++i)
              reinterpret_cast<uint4*>(st_row)[i] = make_uint4(words[4 * i], words[4 * i + 1], words[4 * i + 2],
                                                               words[4 * i + 3]);
            fence_proxy_async_smem();
            bulk_store(static_cast<uint8_t*>(args.out) + static_cast<size_t>(grow) * I + col0, st_row, 64);
            bulk_commit();
            if (g == 0) args.out_scale_t[static_cast<size_t>(nt) * args.capacity + grow] = scale;
          }
        } else {
          // ---- GEMM2 epilogue: routed weight, scatter the row to y[flat]
          const bool real = flat < args.nflat;
          __nv_bfloat16* yrow =
              static_cast<__nv_bfloat16*>(args.out) + static_cast<size_t>(real ? flat : 0) * H + nt * 256 + g * 128;
          if constexpr (kFP8) {
            if (real) {
              uint8_t* st_row = reserve + kSmemReserve + static_cast<size_t>(threadIdx.x - 64) * C::kYPitch;
              bulk_wait_read_all();   // the previous row copy from this staging slot has read it
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = acc_a[16 * c + i] * wt;
                store_bf16x16(reinterpret_cast<__nv_bfloat16*>(st_row + 32 * c), v);
              }
              fence_proxy_async_smem();
              bulk_store(yrow, st_row, 256);
              bulk_commit();
            }
          } else {
            if (!warp_wait(&acc_full[abuf], aphase, abort_flag, args.status, kWhereEpiAcc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t t0 = tmem_base + lane_addr + static_cast<uint32_t>(abuf * C::kAccCols);
            uint32_t packed[64];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float d[16];
              tmem_ld16(t0 + g * 128 + 16 * c, d);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(d[2 * i] * wt, d[2 * i + 1] * wt);
                packed[8 * c + i] = *reinterpret_cast<const uint32_t*>(&h2);
              }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[abuf]);
            if (++abuf == C::kAccBufs) {
              abuf = 0;
              aphase ^= 1u;
            }
            if (real) {
              uint4* dst = reinterpret_cast<uint4*>(yrow);
#pragma unroll
              for (int i = 0; i < 16; ++i)
                dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
            }
          }
        }
      } else {
        // ---------------- swap-AB: row = weight row of the tile, columns = token rows
        constexpr int kHT = C::kHalfTok;           // token columns of this group
        const int tok0 = mb * kBM + g * kHT;       // first sorted row of this group
        float acc_a[kHT];                          // gate (GEMM1) or down (GEMM2)
        float acc_b[kDown ? 1 : kHT];              // up (GEMM1)
        // GEMM2: the tokens' flat ids and routed weights, read before the K loop so that
        // their latency is not on the tile's tail
        constexpr bool kPrefetchRows = kDown && kHT <= 16;
        int flat_j[kPrefetchRows ? kHT : 1];
        float wt_j[kPrefetchRows ? kHT : 1];
        if constexpr (kPrefetchRows) {
#pragma unroll
          for (int j = 0; j < kHT; ++j) flat_j[j] = (*(args.sorted_ids + tok0 + j));
#pragma unroll
          for (int j = 0; j < kHT; ++j) wt_j[j] = flat_j[j] < args.nflat ? route_weight(args.topk_weights, flat_j[j]) : 0.f;
        }
        // column offsets of this group's values inside one accumulator buffer
        const uint32_t col_a = static_cast<uint32_t>(g * kHT);
        const uint32_t col_b = static_cast<uint32_t>(kBM + g * kHT);
        if constexpr (kFP8) {
#pragma unroll
          for (int j = 0; j < kHT; ++j) acc_a[j] = 0.f;
          if constexpr (!kDown) {
#pragma unroll
            for (int j = 0; j < kHT; ++j) acc_b[j] = 0.f;
          }
          const int kb_n = K / 128;
          const float* sw_a;
          const float* sw_b;
          if constexpr (kDown) {
            sw_a = args.w_scale + (static_cast<size_t>(e) * (H / 128) + nt) * kb_n;
            sw_b = sw_a;
          } else {
            sw_a = args.w_scale + (static_cast<size_t>(e) * (2 * I / 128) + nt) * kb_n;
            sw_b = args.w_scale + (static_cast<size_t>(e) * (2 * I / 128) + I / 128 + nt) * kb_n;
          }
          // the scales of K block kb + 1 are loaded right after block kb's drain, so their
          // latency overlaps the wait for the next accumulator instead of following it
          float swa = (*(sw_a + ks0)), swb = (*(sw_b + ks0));
          float fa[kHT];
#pragma unroll
          for (int j = 0; j < kHT; ++j) fa[j] = (*(args.a_scale_t + static_cast<size_t>(ks0) * args.capacity + tok0 + j));
          for (int kb = ks0; kb < ks1; ++kb) {
            if (!warp_wait(&acc_full[abuf], aphase, abort_flag, args.status, kWhereEpiAcc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t t0 = tmem_base + lane_addr + static_cast<uint32_t>(abuf * C::kAccCols);
#pragma unroll
            for (int c = 0; c < kHT / 8; ++c) {
              float da[8], db[8];
              tmem_ld8(t0 + col_a + 8 * c, da);
              if constexpr (!kDown) tmem_ld8(t0 + col_b + 8 * c, db);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                acc_a[8 * c + i] = fmaf(da[i], fa[8 * c + i] * swa, acc_a[8 * c + i]);
                if constexpr (!kDown) acc_b[8 * c + i] = fmaf(db[i], fa[8 * c + i] * swb, acc_b[8 * c + i]);
              }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[abuf]);
            if (kb + 1 < ks1) {
              swa = (*(sw_a + kb + 1));
              swb = (*(sw_b + kb + 1));
              const float* sa_p = args.a_scale_t + static_cast<size_t>(kb + 1) * args.capacity + tok0;
#pragma unroll
              for (int j = 0; j < kHT; ++j) fa[j] = (*(sa_p + j));
            }
            if (++abuf == C::kAccBufs) {
              abuf = 0;
              aphase ^= 1u;
            }
          }
          if (!ok) break;
        } else {
          if (!warp_wait(&acc_full[abuf], aphase, abort_flag, args.status, kWhereEpiAcc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t t0 = tmem_base + lane_addr + static_cast<uint32_t>(abuf * C::kAccCols);
#pragma unroll
          for (int c = 0; c < kHT / 8; ++c) {
            float da[8], db[8];
            tmem_ld8(t0 + col_a + 8 * c, da);
            if constexpr (!kDown) tmem_ld8(t0 + col_b + 8 * c, db);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              acc_a[8 * c + i] = da[i];
              if constexpr (!kDown) acc_b[8 * c + i] = db[i];
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[abuf]);
          if (++abuf == C::kAccBufs) {
            abuf = 0;
            aphase ^= 1u;
          }
        }

        if (splits > 1) {
          // ---- split-K: store this split's fp32 partial sums; the reduce
          // kernel that follows adds the splits in order and runs the epilogue
          constexpr int kAccW = kDown ? kBM : 2 * kBM;
          float* part = args.partials + static_cast<size_t>(unit) * (kAccW * 128);
#pragma unroll
          for (int j = 0; j < kHT; ++j) {
            part[(col_a + j) * 128 + row] = acc_a[j];
            if constexpr (!kDown) part[(col_b + j) * 128 + row] = acc_b[j];
          }
          continue;
        }

        if constexpr (!kDown) {
          // ---- GEMM1: this thread owns intermediate column nt*128 + row for kHT tokens
          const int icol = nt * 128 + row;
#pragma unroll
          for (int j = 0; j < kHT; ++j)
            acc_a[j] = swiglu_bf16(bf16_round(acc_a[j]), bf16_round(acc_b[j]), args.swiglu_limit);
          if constexpr (!kFP8) {
            __nv_bfloat16* a2 = static_cast<__nv_bfloat16*>(args.out);
#pragma unroll
            for (int j = 0; j < kHT; ++j) a2[static_cast<size_t>(tok0 + j) * I + icol] = __float2bfloat16_rn(acc_a[j]);
          } else {
            // amax of each token over the 128 columns: warp butterfly, then the 4 warps of the group
            float* xb = xchg + xbuf * 256;  // [group][quarter][kHT]
#pragma unroll
            for (int j = 0; j < kHT; ++j) {
              float m = fabsf(acc_a[j]);
#pragma unroll
              for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
              if (lane == 0) xb[(g * 4 + q) * kHT + j] = m;
            }
            mbar_arrive(&xchg_bar[xbuf]);
            if (!warp_wait(&xchg_bar[xbuf], xphase, abort_flag, args.status, kWhereEpiXchg)) {
              ok = false;
              break;
            }
            uint8_t* a2 = static_cast<uint8_t*>(args.out);
#pragma unroll
            for (int j = 0; j < kHT; ++j) {
              float m = xb[(g * 4 + 0) * kHT + j];
              m = fmaxf(m, xb[(g * 4 + 1) * kHT + j]);
              m = fmaxf(m, xb[(g * 4 + 2) * kHT + j]);
              m = fmaxf(m, xb[(g * 4 + 3) * kHT + j]);
              const float scale = act_scale_from_amax(m);
              const float v = acc_a[j] * pow2_recip(scale);
              a2[static_cast<size_t>(tok0 + j) * I + icol] =
                  static_cast<uint8_t>(f32x2_to_e4m3x2(v, 0.f) & 0xFFu);
              if (row == 0) args.out_scale_t[static_cast<size_t>(nt) * args.capacity + tok0 + j] = scale;
            }
            xbuf ^= 1;
            if (xbuf == 0) xphase ^= 1u;
          }
        } else {
          // ---- GEMM2: this thread owns H column nt*128 + row for kHT tokens
          __nv_bfloat16* y = static_cast<__nv_bfloat16*>(args.out);
          const int hcol = nt * 128 + row;
#pragma unroll
          for (int j = 0; j < kHT; ++j) {
            if constexpr (kPrefetchRows) {
              if (flat_j[j] < args.nflat)
                y[static_cast<size_t>(flat_j[j]) * H + hcol] = __float2bfloat16_rn(acc_a[j] * wt_j[j]);
            } else {
              const int flat = (*(args.sorted_ids + tok0 + j));
              if (flat < args.nflat)
                y[static_cast<size_t>(flat) * H + hcol] =
                    __float2bfloat16_rn(acc_a[j] * route_weight(args.topk_weights, flat));
            }
          }
        }
      }
    }
    if constexpr (C::kStageY) bulk_wait_all();   // this thread's row copies are complete
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ----------------------------------------------------------------------------
// Split-K reduce for the swap-AB GEMMs.  One CTA of 128 threads per tile;
// thread `row` owns weight row nt*128 + row of the tile for all kBM tokens.
// It adds the S partial sums in split order (deterministic) and runs the
// epilogue the unsplit GEMM would have run: SiLU(gate)*up with bf16 rounding
// (+ per-(token,128) FP8 requantisation, amax over the 128 rows through
// shared memory) for GEMM1, routed weight and scatter to y for GEMM2.
// ----------------------------------------------------------------------------
template <bool kDown, bool kFP8, int kBM>
__global__ void __launch_bounds__(128) splitk_reduce_kernel(Args args) {
  pdl_launch_dependents();
  pdl_wait();
  const int n_tiles = (kDown ? args.H : args.I) / 128;
  const int num_tiles = (*(args.ntpp)) / kBM * n_tiles;
  const int splits = args.splits;
  constexpr int kAccW = kDown ? kBM : 2 * kBM;
  constexpr size_t kUnit = static_cast<size_t>(kAccW) * 128;
  __shared__ float red[4][kBM];
  const int row = threadIdx.x, warp = row >> 5, lane = row & 31;
  for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
    const int mb = tile / n_tiles, nt = tile - mb * n_tiles;
    const int tok0 = mb * kBM;
    const float* part = args.partials + static_cast<size_t>(tile) * splits * kUnit + row;
    float a[kBM], b[kDown ? 1 : kBM];
#pragma unroll
    for (int j = 0; j < kBM; ++j) {
      a[j] = __ldcg(part + j * 128);
      if constexpr (!kDown) b[j] = __ldcg(part + (kBM + j) * 128);
    }
    for (int sp = 1; sp < splits; ++sp) {
      const float* ps = part + sp * kUnit;
#pragma unroll
      for (int j = 0; j < kBM; ++j) {
        a[j] += __ldcg(ps + j * 128);
        if constexpr (!kDown) b[j] += __ldcg(ps + (kBM + j) * 128);
      }
    }
    if constexpr (!kDown) {
      const int icol = nt * 128 + row;
#pragma unroll
      for (int j = 0; j < kBM; ++j) a[j] = swiglu_bf16(bf16_round(a[j]), bf16_round(b[j]), args.swiglu_limit);
      if constexpr (!kFP8) {
        __nv_bfloat16* a2 = static_cast<__nv_bfloat16*>(args.out);
#pragma unroll
        for (int j = 0; j < kBM; ++j) a2[static_cast<size_t>(tok0 + j) * args.I + icol] = __float2bfloat16_rn(a[j]);
      } else {
#pragma unroll
        for (int j = 0; j < kBM; ++j) {
          float m = fabsf(a[j]);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
          if (lane == 0) red[warp][j] = m;
        }
        __syncthreads();
        uint8_t* a2 = static_cast<uint8_t*>(args.out);
#pragma unroll
        for (int j = 0; j < kBM; ++j) {
          const float m = fmaxf(fmaxf(red[0][j], red[1][j]), fmaxf(red[2][j], red[3][j]));
          const float scale = act_scale_from_amax(m);
          a2[static_cast<size_t>(tok0 + j) * args.I + icol] =
              static_cast<uint8_t>(f32x2_to_e4m3x2(a[j] * pow2_recip(scale), 0.f) & 0xFFu);
          if (row == 0) args.out_scale_t[static_cast<size_t>(nt) * args.capacity + tok0 + j] = scale;
        }
        __syncthreads();  // red is reused by the next tile
      }
    } else {
      __nv_bfloat16* y = static_cast<__nv_bfloat16*>(args.out);
      const int hcol = nt * 128 + row;
#pragma unroll
      for (int j = 0; j < kBM; ++j) {
        const int flat = (*(args.sorted_ids + tok0 + j));
        if (flat < args.nflat) {
          const float wt = route_weight(args.topk_weights, flat);
          y[static_cast<size_t>(flat) * args.H + hcol] = __float2bfloat16_rn(a[j] * wt);
        }
      }
    }
  }
}

// ----------------------------------------------------------------------------
// MXFP8 normal tiles ("Hosting von Qwen auf Blackwell", "Quantisierung":
// micro-scaling is what Blackwell's tensor cores consume natively).
//
// tcgen05.mma kind::mxf8f6f4.block_scale: the E8M0 scale of every 32-element K
// block is applied inside the MMA, so the accumulator stays in TMEM for the
// whole K loop -- no per-K-block promotion.  Per K block the producer loads
// the 128 x 128 token tile, the 256 x 128 weight tile (two 128-row boxes for
// GEMM1: gate and up) and three 512-byte SF atoms (tokens; two weight row
// blocks); the MMA thread copies the atoms into TMEM (tcgen05.cp 32x128b,
// replicated to the four lane quarters; 16 columns per stage) and issues four
// K=32 MMAs whose scale-factor byte id walks the atom's four K blocks.
// TMEM: one 256-column accumulator + 4 x 16 SF columns.  The epilogue reads
// its whole share of the accumulator into registers, releases TMEM at once
// (the next tile's MMAs start) and then runs SiLU*up + MX requantisation
// (GEMM1) or the routed weight + scatter (GEMM2).
// ----------------------------------------------------------------------------
template <bool kDown>
struct CfgMx {
  static constexpr int kTokBytes = 128 * 128;
  static constexpr int kWBytes = 256 * 128;
  static constexpr int kSfOffset = kTokBytes + kWBytes;  // three 512-byte atoms
  static constexpr int kStageBytes = 51200;              // 48 KB + 1.5 KB, kept 1024-aligned
  static constexpr int kStages = 4;
  static constexpr int kAccCols = 256;
  static constexpr int kSfCol0 = 256;                    // stage s: columns kSfCol0 + 16 s + [0, 12)
  static constexpr int kTmemCols = 512;
  static constexpr int kTileN = kDown ? 256 : 128;       // output columns per tile
  static constexpr size_t kSmemBytes = static_cast<size_t>(kStages) * kStageBytes + kSmemReserve + 1024;
  static_assert(kSfOffset + 3 * 512 <= kStageBytes, "stage layout");
  static_assert(kSmemBytes <= static_cast<size_t>(kSmemLimit), "shared memory");
};

template <bool kDown>
__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_mx_kernel(const __grid_constant__ CUtensorMap tm_tok, const __grid_constant__ CUtensorMap tm_w,
                       const Args args) {
  using C = CfgMx<kDown>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* reserve = smem + static_cast<size_t>(C::kStages) * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(reserve);
  uint64_t* empty = full + C::kStages;
  uint64_t* acc_full = empty + C::kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_tok);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  const int H = args.H, I = args.I;
  const int K = kDown ? I : H;
  const int kb_n = K / 128;
  const int n_tiles = (kDown ? H : I) / C::kTileN;
  const int num_tiles = ((*(args.ntpp)) / 128) * n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    // All lanes stage the tile's token row ids (GEMM1 gathers code rows of
    // the per-token quantised x); lane 0 issues every copy.
    int32_t* tok_rows = reinterpret_cast<int32_t*>(reserve + kTokRowsOffset);
    const uint64_t pol_w = policy_evict_normal();   // reused by every 128-row block of the expert
    const uint64_t pol_a = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    long long fills = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int mb = tile / n_tiles, nt = tile - mb * n_tiles;
      if (args.gather_tok) {
        for (int i = lane; i < 128; i += 32) {
          const int f = (*(args.sorted_ids + mb * 128 + i));
          tok_rows[i] = f < args.nflat ? f / args.topk : 0;  // padding rows read any valid row
        }
      }
      __syncwarp();
      if (lane == 0) {
        const int e = (*(args.expert_ids + mb));
        // weight rows of the two 128-row blocks of this tile (global row index in [E * Nw, K])
        int w_row0, w_row1;
        if constexpr (kDown) {
          w_row0 = e * H + nt * 256;
          w_row1 = w_row0 + 128;
        } else {
          w_row0 = e * 2 * I + nt * 128;  // gate rows
          w_row1 = w_row0 + I;            // up rows
        }
        const uint8_t* sfa = args.a_sf + static_cast<size_t>(mb) * kb_n * 512;
        const uint8_t* sfb0 = args.w_sf + static_cast<size_t>(w_row0 / 128) * kb_n * 512;
        const uint8_t* sfb1 = args.w_sf + static_cast<size_t>(w_row1 / 128) * kb_n * 512;
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, args.status,
                         MOE_STATUS_WAIT_TIMEOUT | kWhereProducer)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + static_cast<size_t>(stage) * C::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], C::kTokBytes + C::kWBytes + 3 * 512);
          const int kx = kb * 128;
          if (args.gather_tok) {
#pragma unroll 4
            for (int g = 0; g < 32; ++g) {
              const int4 r4 = reinterpret_cast<const int4*>(tok_rows)[g];
              tma_gather4(st + 512 * g, &tm_tok, &full[stage], kx, r4.x, r4.y, r4.z, r4.w);
            }
          } else {
            tma_load_2d(st, &tm_tok, &full[stage], kx, mb * 128, pol_a);
          }
          if constexpr (kDown) {
            tma_load_2d(st + C::kTokBytes, &tm_w, &full[stage], kx, w_row0, pol_w);
          } else {
            tma_load_2d(st + C::kTokBytes, &tm_w, &full[stage], kx, w_row0, pol_w);
            tma_load_2d(st + C::kTokBytes + 16384, &tm_w, &full[stage], kx, w_row1, pol_w);
          }
          bulk_load(st + C::kSfOffset, sfa + static_cast<size_t>(kb) * 512, 512, &full[stage]);
          bulk_load(st + C::kSfOffset + 512, sfb0 + static_cast<size_t>(kb) * 512, 512, &full[stage]);
          bulk_load(st + C::kSfOffset + 1024, sfb1 + static_cast<size_t>(kb) * 512, 512, &full[stage]);
          ++fills;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      __syncwarp();  // the row ids are rewritten only after lane 0 issued this tile's loads
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0 && !ok) {
      // let every copy already issued land before the CTA tears down
      for (int s = 0; s < C::kStages; ++s) {
        const long long n_s = fills / C::kStages + (s < fills % C::kStages ? 1 : 0);
        if (n_s > 0) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[s], static_cast<uint32_t>((n_s - 1) & 1)) &&
                 globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(acc_empty, aphase ^ 1u, abort_flag, args.status, MOE_STATUS_WAIT_TIMEOUT | kWhereMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, args.status, MOE_STATUS_WAIT_TIMEOUT | kWhereMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + static_cast<size_t>(stage) * C::kStageBytes);
          const uint32_t sf_t = tmem_base + static_cast<uint32_t>(C::kSfCol0 + 16 * stage);
          tmem_cp_sf_atom(sf_t, smem_desc_sf_atom(st + C::kSfOffset));
          tmem_cp_sf_atom(sf_t + 4, smem_desc_sf_atom(st + C::kSfOffset + 512));
          tmem_cp_sf_atom(sf_t + 8, smem_desc_sf_atom(st + C::kSfOffset + 1024));
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t koff = k * 32;  // 32 E4M3 elements
            const uint32_t sel = static_cast<uint32_t>(k) << 30;
            mma_mxf8(tmem_base, smem_desc_sw128(st + koff), smem_desc_sw128(st + C::kTokBytes + koff),
                     make_idesc_mx(128, 256, k), (kb > 0 || k > 0) ? 1u : 0u, sf_t | sel, (sf_t + 4) | sel);
          }
          mma_commit(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(acc_full);
        aphase ^= 1u;
      }
      mma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0)) {
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
          report_status(args.status, MOE_STATUS_WAIT_TIMEOUT | kWhereDrain);
          break;
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int g = (warp - 2) >> 2;
    const int row = 32 * q + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    uint32_t aphase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mb = tile / n_tiles, nt = tile - mb * n_tiles;
      const int grow = mb * 128 + row;
      if (!warp_wait(acc_full, aphase, abort_flag, args.status, kWhereEpiAcc)) break;
      aphase ^= 1u;
      tc_fence_after();
      float v[128];  // GEMM1: gate [0, 64) and up [64, 128) of this group; GEMM2: 128 output columns
      const uint32_t t0 = tmem_base + lane_addr;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float a[16], b[16];
        tmem_ld16(t0 + (kDown ? g * 128 + 16 * c : g * 64 + 16 * c), a);
        tmem_ld16(t0 + (kDown ? g * 128 + 64 + 16 * c : 128 + g * 64 + 16 * c), b);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          v[16 * c + i] = a[i];
          v[64 + 16 * c + i] = b[i];
        }
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);  // the next tile's MMAs may overwrite the accumulator now
      if constexpr (!kDown) {
        // SiLU(gate) * up (bf16 rounding points as the oracle), MX requant per 32 columns
        const int col0 = nt * 128 + g * 64;
        uint8_t* dst = static_cast<uint8_t*>(args.out) + static_cast<size_t>(grow) * I + col0;
        uint8_t e8[2];
#pragma unroll
        for (int grp = 0; grp < 2; ++grp) {
          float p[32];
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            p[i] = swiglu_bf16(bf16_round(v[32 * grp + i]), bf16_round(v[64 + 32 * grp + i]), args.swiglu_limit);
            amax = fmaxf(amax, fabsf(p[i]));
          }
          const float scale = act_scale_from_amax(amax);
          const float inv = pow2_recip(scale);
          uint32_t wds[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            wds[i] = static_cast<uint32_t>(f32x2_to_e4m3x2(p[4 * i] * inv, p[4 * i + 1] * inv)) |
                     (static_cast<uint32_t>(f32x2_to_e4m3x2(p[4 * i + 2] * inv, p[4 * i + 3] * inv)) << 16);
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * grp);
          d4[0] = make_uint4(wds[0], wds[1], wds[2], wds[3]);
          d4[1] = make_uint4(wds[4], wds[5], wds[6], wds[7]);
          e8[grp] = e8m0_of_pow2(scale);
        }
        *reinterpret_cast<uint16_t*>(args.out_sf + sf_atom_offset(grow, col0, I)) =
            static_cast<uint16_t>(e8[0] | (static_cast<uint16_t>(e8[1]) << 8));
      } else {
        // routed weight, scatter the row to y[flat]
        const int flat = (*(args.sorted_ids + grow));
        if (flat < args.nflat) {
          const float wt = route_weight(args.topk_weights, flat);
          __nv_bfloat16* yrow = static_cast<__nv_bfloat16*>(args.out) + static_cast<size_t>(flat) * H + nt * 256 +
                                g * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float o[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = v[16 * c + i] * wt;
            store_bf16x16(yrow + 16 * c, o);
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D K-major tensor map: [rows, cols] elements of `elem_bytes`, box = 128 bytes x box_rows, 128-byte swizzle
bool make_map(CUtensorMap* map, const void* base, long long rows, long long cols, int elem_bytes, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const CUtensorMapDataType dt =
      elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * elem_bytes};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool kDown, bool kFP8, bool kSwap, int kBM>
cudaError_t launch_on(const GemmProblem& p, const void* tok, const void* w, const Args& args, cudaStream_t s) {
  using C = Cfg<kDown, kFP8, kSwap, kBM>;
  auto kern = moe_gemm_kernel<kDown, kFP8, kSwap, kBM>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(C::kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int elem = kFP8 ? 1 : 2;
  const long long K = kDown ? p.I : p.H;
  const long long wrows = kDown ? static_cast<long long>(p.E) * p.H : static_cast<long long>(p.E) * 2 * p.I;
  CUtensorMap tm_tok, tm_w;
  // GEMM1 gathers token rows (one-row boxes, tile::gather4) from [T, K]; GEMM2 reads sorted a2 tiles
  if (args.gather_tok ? !make_map(&tm_tok, tok, p.T, K, elem, 1)
                      : !make_map(&tm_tok, tok, p.capacity, K, elem, C::kTokRows))
    return cudaErrorInvalidValue;
  if (!make_map(&tm_w, w, wrows, K, elem, kDown ? C::kWRows : 128)) return cudaErrorInvalidValue;
  const int n_tiles = (kDown ? p.H : p.I) / C::kTileN;
  const long long max_tiles = static_cast<long long>(p.capacity / C::kTokRows) * n_tiles;
  int grid = p.num_sms;
  if (kSwap && p.split_mode == 0) {
    Args a = args;
    a.splits = choose_splits(max_tiles, p.num_sms, static_cast<int>(K / C::kKElems));
    if (max_tiles * a.splits < grid) grid = static_cast<int>(max_tiles * a.splits);
    if (grid <= 0) return cudaSuccess;
    cudaError_t e = launch_pdl(kern, grid, kThreads, C::kSmemBytes, s, tm_tok, tm_w, a);
    if (e != cudaSuccess || a.splits == 1) return e;
    return launch_pdl(splitk_reduce_kernel<kDown, kFP8, kBM>, static_cast<int>(max_tiles), 128, 0, s, a);
  }
  if (max_tiles < grid) grid = static_cast<int>(max_tiles);
  if (grid <= 0) return cudaSuccess;
  Args a = args;
  a.splits = 1;
  return launch_pdl(kern, grid, kThreads, C::kSmemBytes, s, tm_tok, tm_w, a);
}

template <bool kDown>
cudaError_t launch_mx(const GemmProblem& p, const void* tok, const void* w, const Args& args, cudaStream_t s) {
  using C = CfgMx<kDown>;
  auto kern = moe_gemm_mx_kernel<kDown>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(C::kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const long long K = kDown ? p.I : p.H;
  const long long wrows = kDown ? static_cast<long long>(p.E) * p.H : static_cast<long long>(p.E) * 2 * p.I;
  CUtensorMap tm_tok, tm_w;
  if (args.gather_tok ? !make_map(&tm_tok, tok, p.T, K, 1, 1) : !make_map(&tm_tok, tok, p.capacity, K, 1, 128))
    return cudaErrorInvalidValue;
  if (!make_map(&tm_w, w, wrows, K, 1, kDown ? 256 : 128)) return cudaErrorInvalidValue;
  const int n_tiles = (kDown ? p.H : p.I) / C::kTileN;
  const long long max_tiles = static_cast<long long>(p.capacity / 128) * n_tiles;
  int grid = p.num_sms;
  if (max_tiles < grid) grid = static_cast<int>(max_tiles);
  if (grid <= 0) return cudaSuccess;
  return launch_pdl(kern, grid, kThreads, C::kSmemBytes, s, tm_tok, tm_w, args);
}

template <bool kDown, bool kFP8>
cudaError_t dispatch(const GemmProblem& p, const void* tok, const void* w, const Args& args, cudaStream_t s) {
  if constexpr (kFP8) {
    if (p.mx) return launch_mx<kDown>(p, tok, w, args, s);
  }
  if (!p.swap) return launch_on<kDown, kFP8, false, 128>(p, tok, w, args, s);
  switch (p.block_m) {
    case 16: return launch_on<kDown, kFP8, true, 16>(p, tok, w, args, s);
    case 32: return launch_on<kDown, kFP8, true, 32>(p, tok, w, args, s);
    case 64: return launch_on<kDown, kFP8, true, 64>(p, tok, w, args, s);
    default: return cudaErrorInvalidValue;
  }
}

template <bool kDown, bool kFP8, bool kSwap, int kBM>
size_t smem_of() {
  return Cfg<kDown, kFP8, kSwap, kBM>::kSmemBytes;
}

}  // namespace

bool make_tma_map_2d(CUtensorMap* map, const void* base, long long rows, long long cols, int elem_bytes,
                     int box_rows) {
  return make_map(map, base, rows, cols, elem_bytes, box_rows);
}

cudaError_t launch_gemm1(const GemmProblem& p, const void* a1, const void* a1_scale, const void* w13,
                         const void* w13_scale, void* a2, void* a2_scale, cudaStream_t stream) {
  Args args{};
  args.E = p.E;
  args.H = p.H;
  args.I = p.I;
  args.nflat = p.nflat;
  args.capacity = p.capacity;
  args.ntpp = p.ntpp;
  args.expert_ids = p.expert_ids;
  args.sorted_ids = p.sorted_ids;
  args.topk_weights = p.weight_on_input ? nullptr : p.topk_weights;
  args.swiglu_limit = p.swiglu_limit;
  args.gather_tok = p.gather_tok ? 1 : 0;
  args.topk = p.topk;
  if (p.mx) {
    args.a_sf = static_cast<const uint8_t*>(a1_scale);
    args.w_sf = static_cast<const uint8_t*>(w13_scale);
    args.out_sf = static_cast<uint8_t*>(a2_scale);
  } else {
    args.a_scale_t = static_cast<const float*>(a1_scale);
    args.w_scale = static_cast<const float*>(w13_scale);
    args.out_scale_t = static_cast<float*>(a2_scale);
  }
  args.out = a2;
  args.status = p.status;
  args.partials = p.partials;
  args.splits = 1;
  return p.fp8 ? dispatch<false, true>(p, a1, w13, args, stream) : dispatch<false, false>(p, a1, w13, args, stream);
}

cudaError_t launch_gemm2(const GemmProblem& p, const void* a2, const void* a2_scale, const void* w2,
                         const void* w2_scale, void* y, cudaStream_t stream) {
  Args args{};
  args.E = p.E;
  args.H = p.H;
  args.I = p.I;
  args.nflat = p.nflat;
  args.capacity = p.capacity;
  args.ntpp = p.ntpp;
  args.expert_ids = p.expert_ids;
  args.sorted_ids = p.sorted_ids;
  args.topk_weights = p.weight_on_input ? nullptr : p.topk_weights;
  args.swiglu_limit = p.swiglu_limit;
  if (p.mx) {
    args.a_sf = static_cast<const uint8_t*>(a2_scale);
    args.w_sf = static_cast<const uint8_t*>(w2_scale);
  } else {
    args.a_scale_t = static_cast<const float*>(a2_scale);
    args.w_scale = static_cast<const float*>(w2_scale);
  }
  args.out = y;
  args.out_scale_t = nullptr;
  args.status = p.status;
  args.partials = p.partials;
  args.splits = 1;
  return p.fp8 ? dispatch<true, true>(p, a2, w2, args, stream) : dispatch<true, false>(p, a2, w2, args, stream);
}

size_t gemm_smem_bytes(bool gemm2, bool fp8, bool swap, int block_m) {
  if (!swap) {
    if (gemm2) return fp8 ? smem_of<true, true, false, 128>() : smem_of<true, false, false, 128>();
    return fp8 ? smem_of<false, true, false, 128>() : smem_of<false, false, false, 128>();
  }
  return 0;
}

}  // namespace moe
