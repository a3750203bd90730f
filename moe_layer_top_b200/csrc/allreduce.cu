// Fused combine + all-reduce of the expert-parallel layer.
//
// "Hosting von Qwen auf Blackwell" (perplexity.ai), section "MoE Dispatch -
// Combine", "Experten-Parallel": the combine first accumulates, per token,
// the contributions of the experts on this rank, then all-reduces over the
// ranks; section "All-Reduce": instead of every rank loading every peer's
// whole buffer, the buffer is split over the ranks, each reduces its part and
// sends the result to the others.  One kernel does both steps over peer
// memory (plain loads and stores through the peer mappings; no TMA, no
// multicast), so no separate combine launch and no collective library call
// sits between GEMM2 and the next layer:
//
//   1. local accumulation: for every token chunk, partial[t] = bf16(sum of the
//      rank's rows y[t*topk + j] that exist here), j ascending in fp32; the
//      chunk is published by a system-scope release of flags[c] = epoch;
//   2. reduce + broadcast: chunk c belongs to rank c % world; its owner waits
//      (acquire) until every rank published c, sums the ranks' partials in
//      rank order in fp32, rounds once to bf16, stores the result into every
//      rank's out and releases flags[chunks + c] = epoch on every rank;
//   3. the kernel returns once every chunk of this rank's out is done.
//
// Reduce-scatter form (data parallel + expert parallel: every rank brings its
// own T tokens, the layer runs on the ranks' gathered batch of world * T
// tokens, and each rank keeps the rows of its own tokens): the partial covers
// the whole gathered batch, the chunks of rank r's rows belong to rank r, and
// the owner stores the sum into its own out [T, H] only.  The done flags
// still go to every rank: they tell a rank that its partial has been read.
//
// Flags hold the epoch of the last call that passed them (the caller counts
// calls from 1 and zeroes the flags once), so nothing is reset between
// calls.  A rank cannot start call e+1 before its call e returned, i.e. before
// every owner finished reading its partial of call e.
//
// Every wait is bounded (caller's limit, %globaltimer); a wait that runs out
// records MOE_STATUS_WAIT_TIMEOUT | site in the rank's status word and the
// epoch in the rank's abort word (the last flag), after which the rank's other
// waits give up at once, so the kernel always returns.  The
// CTAs of one rank wait on one another (phase 2 on phase 1), so each rank's
// grid is a cooperative launch (all CTAs resident).
#include <cuda_bf16.h>

#include "allreduce.h"
#include "common.cuh"

namespace moe {

namespace {

constexpr int kThreadsAr = 256;
constexpr int kWhereArReady = 0x31, kWhereArDone = 0x32;

struct ArParams {
  AllreduceRank r[kMaxRanks];
  int world, rank, topk, H, chunk_tokens, ctas_per_rank;
  int scatter;        // 0: all-reduce of [rows, H]; 1: reduce-scatter of [world * rows, H]
  int rows;           // rows of out (per rank)
  int nchunks_rows;   // chunks of `rows` rows
  int nchunks;        // all chunks: nchunks_rows, or world * nchunks_rows when scattering
  uint32_t epoch;
  unsigned long long timeout_ns;
};

// token rows [t0, t1) of chunk c in the partial buffers
__device__ __forceinline__ void chunk_rows(const ArParams& P, int c, long long& t0, long long& t1) {
  const int region = P.scatter ? c / P.nchunks_rows : 0;
  const int local = P.scatter ? c - region * P.nchunks_rows : c;
  const long long base = static_cast<long long>(region) * P.rows;
  t0 = base + static_cast<long long>(local) * P.chunk_tokens;
  t1 = t0 + P.chunk_tokens;
  if (t1 > base + P.rows) t1 = base + P.rows;
}

struct alignas(16) bf16x8 {
  __nv_bfloat162 h[4];
};

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const bf16x8 b = *reinterpret_cast<const bf16x8*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(b.h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  bf16x8 b;
#pragma unroll
  for (int i = 0; i < 4; ++i) b.h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return *reinterpret_cast<const uint4*>(&b);
}

__device__ __forceinline__ void st_release_sys(int* p, int v) {
  asm volatile("st.release.sys.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire_sys(const int* p) {
  int v;
  asm volatile("ld.acquire.sys.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// 16 bytes through L2 only (a peer's partial, written during this launch)
__device__ __forceinline__ uint4 ld_cg_v4(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

__device__ __forceinline__ bool reached(int v, uint32_t epoch) {
  return static_cast<int>(static_cast<uint32_t>(v) - epoch) >= 0;
}

// one thread: bounded wait until *flag has reached this call's epoch; false
// at once when the rank already gave up in this call (abort word = epoch)
__device__ bool wait_epoch(const int* flag, uint32_t epoch, int* abort_word, int* status,
                           unsigned long long timeout_ns, int where) {
  volatile int* ab = abort_word;
  if (reached(ld_acquire_sys(flag), epoch)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (reached(ld_acquire_sys(flag), epoch)) return true;
    if (reached(*ab, epoch)) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      report_status(status, MOE_STATUS_WAIT_TIMEOUT | where);
      *ab = static_cast<int>(epoch);
      return false;
    }
    __nanosleep(64);
  }
}

__global__ void __launch_bounds__(kThreadsAr) combine_allreduce_kernel(const ArParams P) {
  __shared__ int ok;
  const bool emulated = P.rank < 0;
  const int me = emulated ? static_cast<int>(blockIdx.x) / P.ctas_per_rank : P.rank;
  const int cta = emulated ? static_cast<int>(blockIdx.x) % P.ctas_per_rank : static_cast<int>(blockIdx.x);
  const AllreduceRank& R = P.r[me];
  const int vecs = P.H / 8;
  const uint4* y = static_cast<const uint4*>(R.y);
  uint4* partial = static_cast<uint4*>(R.partial);
  int* abort_word = R.flags + 2 * P.nchunks;

  // 1. local accumulation of this CTA's chunks, each published when written
  for (int c = cta; c < P.nchunks; c += P.ctas_per_rank) {
    long long t0, t1;
    chunk_rows(P, c, t0, t1);
    const long long n = (t1 - t0) * vecs;
    for (long long i = threadIdx.x; i < n; i += kThreadsAr) {
      const long long t = t0 + i / vecs;
      const int v = static_cast<int>(i % vecs);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int j = 0; j < P.topk; ++j) {
        const long long f = t * P.topk + j;
        if (R.pos_of_flat && R.pos_of_flat[f] < 0) continue;  // another rank's expert: no row here
        float g[8];
        unpack8(y[f * vecs + v], g);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] += g[q];
      }
      partial[t * vecs + v] = pack8(acc);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence_system();
      st_release_sys(R.flags + c, static_cast<int>(P.epoch));
    }
  }

  // 2. this rank's chunks: every rank's partial -> sum -> every rank's out (all-reduce) or this
  //    rank's out (reduce-scatter)
  const int c_first = P.scatter ? me * P.nchunks_rows : me;
  const int c_end = P.scatter ? (me + 1) * P.nchunks_rows : P.nchunks;
  const int c_step = P.scatter ? 1 : P.world;
  const long long out_base = P.scatter ? static_cast<long long>(me) * P.rows * vecs : 0;
  int k = 0;
  for (int c = c_first; c < c_end; c += c_step, ++k) {
    if (k % P.ctas_per_rank != cta) continue;
    if (threadIdx.x == 0) {
      bool good = true;
      for (int p = 0; p < P.world && good; ++p)
        good = wait_epoch(P.r[p].flags + c, P.epoch, abort_word, R.status, P.timeout_ns, kWhereArReady);
      ok = good ? 1 : 0;
    }
    __syncthreads();
    if (ok) {
      long long t0, t1;
      chunk_rows(P, c, t0, t1);
      const long long n = (t1 - t0) * vecs;
      for (long long i = threadIdx.x; i < n; i += kThreadsAr) {
        const long long e = t0 * vecs + i;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int p = 0; p < P.world; ++p) {
          float g[8];
          unpack8(ld_cg_v4(static_cast<const uint4*>(P.r[p].partial) + e), g);
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[q] += g[q];
        }
        const uint4 o = pack8(acc);
        if (P.scatter)
          static_cast<uint4*>(R.out)[e - out_base] = o;
        else
          for (int p = 0; p < P.world; ++p) static_cast<uint4*>(P.r[p].out)[e] = o;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0 && ok) {
      __threadfence_system();
      for (int p = 0; p < P.world; ++p) st_release_sys(P.r[p].flags + P.nchunks + c, static_cast<int>(P.epoch));
    }
    __syncthreads();  // ok is rewritten for the next chunk
  }

  // 3. return once every chunk has been reduced: this rank's out is complete and no owner still
  //    reads its partial
  if (threadIdx.x == 0) {
    for (int c = cta; c < P.nchunks; c += P.ctas_per_rank)
      if (!wait_epoch(R.flags + P.nchunks + c, P.epoch, abort_word, R.status, P.timeout_ns, kWhereArDone)) break;
  }
}

}  // namespace

AllreduceChunks allreduce_chunks(int T, int world, bool scatter) {
  if (scatter) {
    // chunks of each rank's rows; the world regions together stay within kMaxArChunks
    if (T <= 0) return {1, 0};
    long long target = 64;
    if (target * world > kMaxArChunks) target = kMaxArChunks / world;
    if (target > T) target = T;
    const int ct = static_cast<int>((T + target - 1) / target);
    return {ct, world * ((T + ct - 1) / ct)};
  }
  if (T <= 0) return {1, 0};
  long long target = 64LL * world;  // a few chunks per CTA of every rank at decode sizes
  if (target > kMaxArChunks) target = kMaxArChunks;
  if (target > T) target = T;
  const int ct = static_cast<int>((T + target - 1) / target);
  return {ct, (T + ct - 1) / ct};
}

cudaError_t launch_combine_allreduce(const AllreduceRank* ranks, int world, int rank, int T, int topk, int H,
                                     bool scatter, uint32_t epoch, unsigned long long timeout_ns, int num_sms,
                                     cudaStream_t stream) {
  const AllreduceChunks ch = allreduce_chunks(T, world, scatter);
  if (ch.nchunks == 0) return cudaSuccess;
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, combine_allreduce_kernel, kThreadsAr, 0);
  if (e != cudaSuccess) return e;
  const int resident = per_sm * num_sms;
  const int grids = rank < 0 ? world : 1;  // the emulated launch holds every rank's CTAs
  int ctas = resident / grids;
  if (ctas > num_sms) ctas = num_sms;
  if (ctas > ch.nchunks) ctas = ch.nchunks;
  if (ctas < 1) return cudaErrorCooperativeLaunchTooLarge;
  ArParams P{};
  for (int p = 0; p < world; ++p) P.r[p] = ranks[p];
  P.world = world;
  P.rank = rank;
  P.topk = topk;
  P.H = H;
  P.chunk_tokens = ch.chunk_tokens;
  P.scatter = scatter ? 1 : 0;
  P.rows = T;
  P.nchunks = ch.nchunks;
  P.nchunks_rows = scatter ? ch.nchunks / world : ch.nchunks;
  P.ctas_per_rank = ctas;
  P.epoch = epoch;
  P.timeout_ns = timeout_ns;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas * grids));
  cfg.blockDim = dim3(kThreadsAr);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // a rank's CTAs wait on one another
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_allreduce_kernel, P);
}

}  // namespace moe
