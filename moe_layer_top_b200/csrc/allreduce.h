// Host-side launcher of the fused combine + all-reduce of expert parallelism
// (internal to the library; see allreduce.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kMaxRanks = 16;       // one NVLink domain of the sizes the pages use (EP = 4 ... 16)
constexpr int kMaxArChunks = 1024;  // token chunks per call (flags: 2 ints per chunk and rank)

// One rank's buffers, as mapped in the calling process (a peer's through its
// peer mapping).  All bf16 arrays are row-major with rows of H elements.
struct AllreduceRank {
  // (sizes for the all-reduce; the reduce-scatter form has world * T rows in y, pos_of_flat and partial)
  const void* y;               // bf16 [T*topk, H]: the rank's GEMM2 rows (read by that rank only)
  const int32_t* pos_of_flat;  // int32 [T*topk]: -1 = the assignment has no row on that rank (NULL: all have)
  void* partial;               // bf16 [T, H]: the rank's local sums (read by every rank)
  void* out;                   // bf16 [T, H]: the layer (written by every rank; reduce-scatter: by the rank)
  int* flags;                  // int32 [2 * chunks + 1]: chunk ready / chunk done epochs, abort epoch
  int* status;                 // int32 status word of the rank
};

struct AllreduceChunks {
  int chunk_tokens;
  int nchunks;
};

// Token chunking of a call: the same on every rank (it depends on T, world and the form only).
// Reduce-scatter: T = rows per rank; nchunks counts the chunks of all world regions.
AllreduceChunks allreduce_chunks(int T, int world, bool scatter);

// rank >= 0: this rank's kernel (its peers launch theirs at the same time on
// their GPUs); rank < 0: every rank's part in one cooperative launch on this
// device (all buffers local), which is how the exchange is tested on one GPU.
// scatter: reduce-scatter form -- partial [world * T, H], out [T, H] per rank.
cudaError_t launch_combine_allreduce(const AllreduceRank* ranks, int world, int rank, int T, int topk, int H,
                                     bool scatter, uint32_t epoch, unsigned long long timeout_ns, int num_sms,
                                     cudaStream_t stream);

}  // namespace moe
