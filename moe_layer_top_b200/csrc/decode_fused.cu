// Persistent decode kernel: the whole bf16 layer for a small batch in ONE
// cooperative launch -- route, align, GEMM1 + SiLU*up, GEMM2 + routed weight,
// combine -- so that no kernel boundary sits between the phases.
//
// Phases (all CTAs resident; every cross-CTA wait is bounded):
//   0. CTA 0 routes the T tokens (one warp per token, "Warum MoE-Kernel so
//      wichtig sind", AWS/kinachrichten page: token routing) and aligns the
//      T*topk <= 256 assignments in shared memory (stable rank by a direct
//      count over the earlier assignments, padded offsets, sentinel padding:
//      the same sorted_token_ids / expert_ids as the align kernels), writes
//      them out and publishes a flag; the other CTAs wait for it.
//   1. One stream of units per CTA: first the GEMM1 tiles (expert block of 16
//      token rows x 128 intermediate columns, swap-AB: the 128 gate and 128
//      up weight rows fill the MMA M, the tokens its N; token rows gathered
//      from x with TMA tile::gather4), then the GEMM2 tiles (16 rows x 128
//      output columns).  A GEMM1 tile's epilogue stores its a2 columns and
//      bumps ready[block]; a GEMM2 tile's producer waits until ready[block]
//      counts all I/128 GEMM1 tiles of its block, then TMA-loads the a2 rows.
//      Every CTA issues all its GEMM1 work before any GEMM2 wait, so the waits
//      always end.
//   2. When all GEMM2 tiles are counted, every CTA combines a slice of the
//      output rows: out[t] = bf16(sum_j y[t*topk + j]).
#include "common.cuh"
#include "kernels.h"
#include "router.cuh"

namespace moe {

namespace {

constexpr int kBM = kDecodeBlockM;        // token rows per expert block = MMA N
constexpr int kStages = 6;
constexpr int kTokBytes = kBM * 128;      // 16 rows x 64 bf16
constexpr int kWBytes = 256 * 128;        // GEMM1: 128 gate + 128 up rows (GEMM2 uses 128 rows)
constexpr int kStageBytes = kTokBytes + kWBytes;
constexpr int kReserve = 4096;
constexpr size_t kSmemBytes = static_cast<size_t>(kStages) * kStageBytes + kReserve + 1024;
constexpr int kAccCols = 2 * kBM;         // GEMM1: gate | up (GEMM2 uses the first kBM)
constexpr int kTmemCols = 64;             // two accumulator buffers
constexpr int kThreadsDf = 320;           // producer, MMA, 8 epilogue warps
constexpr int kHT = kBM / 2;              // token columns per epilogue group
constexpr int kTokRowsOff = 3072;         // reserve: the tile's gathered token rows

// sync words (workspace, zeroed before the launch)
constexpr int kSyncAligned = 0, kSyncGemm2Done = 1, kSyncReady = 8;

// wait sites in the status word
constexpr int kWhereAlignFlag = 0x21, kWhereReady = 0x22, kWhereDone = 0x23, kWhereProd = 0x24, kWhereMmaDf = 0x25,
              kWhereEpiDf = 0x26, kWhereDrainDf = 0x27;

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// generic-proxy global writes of this thread ordered with later async-proxy (TMA) accesses
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// bounded wait until *p >= target (gpu-scope acquire); false on timeout or abort
__device__ bool wait_count(const int* p, int target, volatile int* abort, int* status, int where) {
  if (ld_acquire_gpu(p) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (ld_acquire_gpu(p) >= target) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
      *abort = 1;
      report_status(status, MOE_STATUS_WAIT_TIMEOUT | where);
      return false;
    }
    __nanosleep(100);
  }
}

// largest e with offs[e] <= pos: the expert owning padded row pos (empty
// experts share their successor's offset and lose to the higher index)
__device__ __forceinline__ int owner_of(const int32_t* offs, int E, int pos) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offs[mid] <= pos) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Phase 0, CTA 0: route (optional) + align of n <= 256 assignments.
template <int VPL>
__device__ void route_align_cta(const DecodeProblem& p, int32_t* scratch) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = p.T * p.topk, E = p.E;
  int32_t* ids_s = scratch;                      // [256]
  int32_t* rank_s = ids_s + kDecodeMaxAssignments;  // [256]
  int32_t* cnt = rank_s + kDecodeMaxAssignments;    // [256]
  int32_t* offs = cnt + kDecodeMaxExperts;          // [257]
  if (p.logits != nullptr) {
    for (int t = warp; t < p.T; t += kThreadsDf / 32) {
      int id;
      float w;
      route_token<VPL>(p.logits + static_cast<size_t>(t) * E, E, p.topk, p.renormalize, lane, id, w);
      if (lane < p.topk) {
        p.topk_ids[t * p.topk + lane] = id;
        p.topk_weights[t * p.topk + lane] = w;
        ids_s[t * p.topk + lane] = id;
      }
    }
  } else {
    for (int i = tid; i < n; i += kThreadsDf) ids_s[i] = (*(p.ids_in + i));
  }
  for (int e = tid; e < E; e += kThreadsDf) cnt[e] = 0;
  __syncthreads();
  // stable rank: earlier assignments of the same expert (ascending flat order)
  for (int i = tid; i < n; i += kThreadsDf) {
    const int e = ids_s[i];
    if (e < 0 || e >= E) {
      rank_s[i] = -1;
      report_status(p.status, MOE_STATUS_BAD_EXPERT_ID);
      continue;
    }
    int r = 0;
    for (int j = 0; j < i; ++j) r += ids_s[j] == e ? 1 : 0;
    rank_s[i] = r;
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the block-padded counts, 8 experts per lane
    int local[8];
    int sum = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e = lane * 8 + k;
      const int c = e < E ? cnt[e] : 0;
      local[k] = (c + kBM - 1) / kBM * kBM;
      sum += local[k];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    int run = incl - sum;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e = lane * 8 + k;
      if (e < E) offs[e] = run;
      run += local[k];
    }
    if (lane == 31) offs[E] = incl;
  }
  __syncthreads();
  const int ntpp = offs[E];
  for (int i = tid; i < n; i += kThreadsDf)
    if (rank_s[i] >= 0) p.sorted_ids[offs[ids_s[i]] + rank_s[i]] = i;
  for (int pos = tid; pos < p.capacity; pos += kThreadsDf) {
    bool pad = true;
    if (pos < ntpp) {
      const int e = owner_of(offs, E, pos);
      pad = pos >= offs[e] + cnt[e];
    }
    if (pad) p.sorted_ids[pos] = n;
  }
  for (int b = tid; b < p.capacity / kBM; b += kThreadsDf)
    p.expert_ids[b] = b * kBM < ntpp ? owner_of(offs, E, b * kBM) : -1;
  for (int e = tid; e <= E; e += kThreadsDf) {
    p.offsets[e] = offs[e];
    if (e < E) p.counts[e] = cnt[e];
  }
  if (tid == 0) *p.ntpp = ntpp;
}

}  // namespace

namespace {

template <int VPL>
__global__ void __launch_bounds__(kThreadsDf, 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w13,
                        const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_a2,
                        const DecodeProblem p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* reserve = smem + static_cast<size_t>(kStages) * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(reserve);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* tok_rows = reinterpret_cast<int32_t*>(reserve + kTokRowsOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w13);
    tma_prefetch_desc(&tm_w2);
    tma_prefetch_desc(&tm_a2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // ---------------------------------------------------------------- phase 0
  int* sync = p.sync;
  if (blockIdx.x == 0) {
    route_align_cta<VPL>(p, reinterpret_cast<int32_t*>(smem));  // the ring is free until phase 1
    __threadfence();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // TMA overwrites this scratch next
    __syncthreads();
    if (tid == 0) red_release_add(sync + kSyncAligned, 1);
  } else if (tid == 0) {
    wait_count(sync + kSyncAligned, 1, abort_flag, p.status, kWhereAlignFlag);
  }
  __syncthreads();

  const int n = p.T * p.topk;
  const int H = p.H, I = p.I;
  const int nblocks = *abort_flag ? 0 : ld_cg_i32(p.ntpp) / kBM;
  const int nt1 = I / 128, nt2 = H / 128;
  const int U1 = nblocks * nt1, U = U1 + nblocks * nt2;
  const int ks1 = H / 64, ks2 = I / 64;  // bf16: 64 K elements (128 bytes) per stage
  const float* wts = p.logits != nullptr ? p.topk_weights : p.weights_in;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_a = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    long long fills = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
      const bool g1 = u < U1;
      const int v = g1 ? u : u - U1;
      const int mb = v / (g1 ? nt1 : nt2), nt = v - mb * (g1 ? nt1 : nt2);
      if (g1) {
        for (int i = lane; i < kBM; i += 32) {
          const int f = ld_cg_i32(p.sorted_ids + mb * kBM + i);
          tok_rows[i] = f < n ? f / p.topk : 0;  // padding rows read any valid row
        }
      }
      __syncwarp();
      if (lane == 0) {
        const int e = ld_cg_i32(p.expert_ids + mb);
        const int nks = g1 ? ks1 : ks2;
        int ks = 0;
        if (!g1) {
          // GEMM2 tile: its weight tiles go out first (they need only the
          // alignment); the a2 rows follow once all I/128 GEMM1 tiles of the
          // block (8 epilogue warps each) have been published
          int pre_stage[kStages];
          for (; ks < nks && ks < kStages && ok; ++ks) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, MOE_STATUS_WAIT_TIMEOUT | kWhereProd)) {
              ok = false;
              break;
            }
            uint8_t* st = smem + static_cast<size_t>(stage) * kStageBytes;
            mbar_arrive_expect_tx(&full[stage], kTokBytes + 16384);
            tma_load_2d(st + kTokBytes, &tm_w2, &full[stage], ks * 64, e * H + nt * 128, pol_w);
            pre_stage[ks] = stage;
            ++fills;
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (ok) ok = wait_count(sync + kSyncReady + mb, nt1 * 8, abort_flag, p.status, kWhereReady);
          if (ok) {
            fence_proxy_async_global();
            for (int i = 0; i < ks; ++i)
              tma_load_2d(smem + static_cast<size_t>(pre_stage[i]) * kStageBytes, &tm_a2, &full[pre_stage[i]],
                          i * 64, mb * kBM, pol_a);
          }
        }
        for (; ks < nks && ok; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, MOE_STATUS_WAIT_TIMEOUT | kWhereProd)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + static_cast<size_t>(stage) * kStageBytes;
          const int kx = ks * 64;
          if (g1) {
            mbar_arrive_expect_tx(&full[stage], kStageBytes);
#pragma unroll
            for (int q4 = 0; q4 < kBM / 4; ++q4) {
              const int4 r4 = reinterpret_cast<const int4*>(tok_rows)[q4];
              tma_gather4(st + 512 * q4, &tm_x, &full[stage], kx, r4.x, r4.y, r4.z, r4.w);
            }
            const int wr = e * 2 * I + nt * 128;
            tma_load_2d(st + kTokBytes, &tm_w13, &full[stage], kx, wr, pol_w);           // gate rows
            tma_load_2d(st + kTokBytes + 16384, &tm_w13, &full[stage], kx, wr + I, pol_w);  // up rows
          } else {
            mbar_arrive_expect_tx(&full[stage], kTokBytes + 16384);
            tma_load_2d(st, &tm_a2, &full[stage], kx, mb * kBM, pol_a);
            tma_load_2d(st + kTokBytes, &tm_w2, &full[stage], kx, e * H + nt * 128, pol_w);
          }
          ++fills;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      __syncwarp();  // the row ids are rewritten only after lane 0 issued this tile's loads
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0 && !ok) {
      for (int s = 0; s < kStages; ++s) {  // let every copy already issued land
        const long long n_s = fills / kStages + (s < fills % kStages ? 1 : 0);
        if (n_s > 0) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[s], static_cast<uint32_t>((n_s - 1) & 1)) &&
                 globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(128, kBM, false);
      int stage = 0, abuf = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const bool g1 = u < U1;
        const int nks = g1 ? ks1 : ks2;
        if (!mbar_wait(&acc_empty[abuf], aphase ^ 1u, abort_flag, p.status, MOE_STATUS_WAIT_TIMEOUT | kWhereMmaDf))
          break;
        tc_fence_after();
        for (int ks = 0; ks < nks; ++ks) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, MOE_STATUS_WAIT_TIMEOUT | kWhereMmaDf)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(abuf * kAccCols);
          const uint32_t tok = smem_u32(smem + static_cast<size_t>(stage) * kStageBytes);
          const uint32_t w = tok + kTokBytes;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t koff = k * 32;  // 16 bf16
            const uint32_t acc = (ks > 0 || k > 0) ? 1u : 0u;
            const uint64_t bd = smem_desc_sw128(tok + koff);
            mma_bf16(d, smem_desc_sw128(w + koff), bd, idesc, acc);
            if (g1) mma_bf16(d + kBM, smem_desc_sw128(w + 16384 + koff), bd, idesc, acc);
          }
          mma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[abuf]);
        abuf ^= 1;
        if (abuf == 0) aphase ^= 1u;
      }
      mma_commit(drain);  // TMEM must not be freed under a running MMA
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0)) {
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
          report_status(p.status, MOE_STATUS_WAIT_TIMEOUT | kWhereDrainDf);
          break;
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;             // TMEM lane quarter
    const int g = (warp - 2) >> 2;      // token group: columns g*8 .. g*8+7
    const int row = 32 * q + lane;      // weight row of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    __nv_bfloat16* a2 = static_cast<__nv_bfloat16*>(p.a2);
    __nv_bfloat16* y = static_cast<__nv_bfloat16*>(p.y);
    int abuf = 0;
    uint32_t aphase = 0;
    for (int u = blockIdx.x; u < U; u += gridDim.x) {
      const bool g1 = u < U1;
      const int v = g1 ? u : u - U1;
      const int mb = v / (g1 ? nt1 : nt2), nt = v - mb * (g1 ? nt1 : nt2);
      if (!mbar_wait(&acc_full[abuf], aphase, abort_flag, p.status, MOE_STATUS_WAIT_TIMEOUT | kWhereEpiDf)) break;
      tc_fence_after();
      const uint32_t t0 = tmem_base + lane_addr + static_cast<uint32_t>(abuf * kAccCols);
      float va[kHT], vb[kHT];
      tmem_ld8(t0 + g * kHT, va);
      tmem_ld8(t0 + kBM + g * kHT, vb);  // up half (GEMM1); unused columns for GEMM2
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[abuf]);
      abuf ^= 1;
      if (abuf == 0) aphase ^= 1u;
      const int tok0 = mb * kBM + g * kHT;
      if (g1) {
        const int icol = nt * 128 + row;
#pragma unroll
        for (int j = 0; j < kHT; ++j)
          a2[static_cast<size_t>(tok0 + j) * I + icol] =
              __float2bfloat16_rn(swiglu_bf16(bf16_round(va[j]), bf16_round(vb[j]), p.swiglu_limit));
        fence_proxy_async_global();  // these stores are read back by TMA (GEMM2 producers)
      } else {
        const int hcol = nt * 128 + row;
#pragma unroll
        for (int j = 0; j < kHT; ++j) {
          const int flat = ld_cg_i32(p.sorted_ids + tok0 + j);
          if (flat < n) y[static_cast<size_t>(flat) * H + hcol] = __float2bfloat16_rn(va[j] * (*(wts + flat)));
        }
      }
      // publish this warp's part of the tile: the warp barrier orders the lanes'
      // stores before lane 0's gpu-scope release (the counters count warps)
      __syncwarp();
      if (lane == 0) red_release_add(g1 ? sync + kSyncReady + mb : sync + kSyncGemm2Done, 1);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }

  // ---------------------------------------------------------------- phase 2: combine
  if (tid == 0) wait_count(sync + kSyncGemm2Done, (U - U1) * 8, abort_flag, p.status, kWhereDone);
  __syncthreads();
  if (*abort_flag) return;
  const int vecs = H / 8;
  const long long total = static_cast<long long>(p.T) * vecs;
  for (long long i = static_cast<long long>(blockIdx.x) * kThreadsDf + tid; i < total;
       i += static_cast<long long>(gridDim.x) * kThreadsDf) {
    const long long t = i / vecs;
    const int vv = static_cast<int>(i - t * vecs);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < p.topk; ++j) {
      const uint4 u4 = __ldcg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.y) +
                                                             (t * p.topk + j) * H) + vv);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u4);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(h[k]);
        acc[2 * k] += f.x;
        acc[2 * k + 1] += f.y;
      }
    }
    __nv_bfloat162 o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] = __floats2bfloat162_rn(acc[2 * k], acc[2 * k + 1]);
    reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + t * H)[vv] = *reinterpret_cast<const uint4*>(o);
  }
}

}  // namespace

bool decode_fused_fits(int T, int E, int topk, int H, int I) {
  return T >= 1 && static_cast<long long>(T) * topk <= kDecodeMaxAssignments && E <= kDecodeMaxExperts &&
         H % 128 == 0 && I % 128 == 0;
}

cudaError_t launch_decode_fused(const DecodeProblem& p, cudaStream_t stream) {
  auto kern = p.E <= 128 ? decode_fused_kernel<4> : decode_fused_kernel<8>;
  static bool attr_set[2] = {false, false};
  const int idx = p.E <= 128 ? 0 : 1;
  if (!attr_set[idx]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set[idx] = true;
  }
  CUtensorMap tm_x, tm_w13, tm_w2, tm_a2;
  if (!make_tma_map_2d(&tm_x, p.x, p.T, p.H, 2, 1) ||
      !make_tma_map_2d(&tm_w13, p.w13, static_cast<long long>(p.E) * 2 * p.I, p.H, 2, 128) ||
      !make_tma_map_2d(&tm_w2, p.w2, static_cast<long long>(p.E) * p.H, p.I, 2, 128) ||
      !make_tma_map_2d(&tm_a2, p.a2, p.capacity, p.I, 2, kBM))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.num_sms));
  cfg.blockDim = dim3(kThreadsDf);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs resident: the phases wait on one another
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tm_x, tm_w13, tm_w2, tm_a2, p);
}

}  // namespace moe
