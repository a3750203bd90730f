// Memory-bound helpers of the MoE pipeline: preparing GEMM1's token rows
// (per-token FP8 / MXFP8 quantisation with scales scattered to the sorted
// rows, the sorted copy of those code rows for normal tiles, the bf16 gather
// for normal bf16 tiles, the router-weight scaling), the
// top-k combine, and the FP8 128x128 and MXFP8 weight quantisers used when
// weights are prepared.  All move 16-byte vectors per thread.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

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

}  // namespace

// ----------------------------------------------------------------------------
// gather: a1[r] = x[sorted_ids[r] / topk] for the real rows r <
// num_tokens_post_padded; padding rows are not written.  FP8: per (row, 128 columns) the power-of-two
// scale of the vLLM PR #64760 analysis §1.2 rule, codes into a1 [cap, H],
// scales into a1_scale_t [H/128, cap] (K-block major for the GEMM epilogue).
// MXFP8 ("Hosting von Qwen auf Blackwell", "Quantisierung"): the same rule
// per (row, 32 columns), E8M0 scale bytes into the SF-atom layout the
// block-scaled MMA reads.  A block walks rows; a thread owns 8 consecutive
// columns, 16 threads one 128-column group (4 threads one 32-column group).
// ----------------------------------------------------------------------------
// quantisation of the gathered rows
enum GatherQ { kGatherBf16 = 0, kGatherFp8 = 1, kGatherMx = 2 };

template <int Q>
__global__ void __launch_bounds__(256) gather_kernel(const __nv_bfloat16* x, int H, int topk,
                                                     int nflat, const int32_t* sorted_ids,
                                                     const int32_t* ntpp_ptr, int capacity,
                                                     const float* row_weight, void* a1, void* a1_scale) {
  pdl_launch_dependents();
  pdl_wait();
  const int ntpp = *ntpp_ptr;
  const int vecs = H / 8;
  const int iters = (vecs + blockDim.x - 1) / blockDim.x;
  for (int row = blockIdx.x; row < ntpp; row += gridDim.x) {
    const int flat = (*(sorted_ids + row));
    // padding rows are left as they are: every GEMM output row and column
    // depends only on its own input row, and padding outputs are never stored
    if (flat >= nflat) continue;
    const __nv_bfloat16* src = x + static_cast<size_t>(flat / topk) * H;
    // router weight applied on the input: the row is w * x, rounded to bf16
    const float rw = row_weight ? (*(row_weight + flat)) : 1.0f;
    for (int it = 0; it < iters; ++it) {
      const int v = it * blockDim.x + threadIdx.x;  // uniform trip count: shuffles below see full warps
      const bool in = v < vecs;
      uint4 u = make_uint4(0, 0, 0, 0);
      if (in) u = (*(reinterpret_cast<const uint4*>(src) + v));
      if (row_weight) {
        float f[8];
        unpack8(u, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] *= rw;
        u = pack8(f);
      }
      if constexpr (Q == kGatherBf16) {
        if (in) reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a1) + static_cast<size_t>(row) * H)[v] = u;
      } else {
        float f[8];
        unpack8(u, f);
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
        // group of 128 columns = 16 threads (FP8), of 32 columns = 4 threads (MXFP8)
#pragma unroll
        for (int off = (Q == kGatherFp8 ? 8 : 2); off > 0; off >>= 1)
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const float scale = act_scale_from_amax(amax);
        const float inv = pow2_recip(scale);
        uint2 q;
        q.x = static_cast<uint32_t>(f32x2_to_e4m3x2(f[0] * inv, f[1] * inv)) |
              (static_cast<uint32_t>(f32x2_to_e4m3x2(f[2] * inv, f[3] * inv)) << 16);
        q.y = static_cast<uint32_t>(f32x2_to_e4m3x2(f[4] * inv, f[5] * inv)) |
              (static_cast<uint32_t>(f32x2_to_e4m3x2(f[6] * inv, f[7] * inv)) << 16);
        if (in) {
          reinterpret_cast<uint2*>(static_cast<uint8_t*>(a1) + static_cast<size_t>(row) * H)[v] = q;
          if constexpr (Q == kGatherFp8) {
            if ((v & 15) == 0) static_cast<float*>(a1_scale)[static_cast<size_t>(v >> 4) * capacity + row] = scale;
          } else {
            if ((v & 3) == 0) static_cast<uint8_t*>(a1_scale)[sf_atom_offset(row, v * 8, H)] = e8m0_of_pow2(scale);
          }
        }
      }
    }
  }
}

cudaError_t launch_gather(const void* x, int H, int topk, int nflat, const int32_t* sorted_ids,
                          const int32_t* ntpp, int capacity, bool fp8, bool mx, const float* row_weight, void* a1,
                          void* a1_scale, cudaStream_t stream) {
  if (capacity == 0) return cudaSuccess;
  int blocks = capacity < 148 * 8 ? capacity : 148 * 8;
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (mx)
    return launch_pdl(gather_kernel<kGatherMx>, blocks, 256, 0, stream, xb, H, topk, nflat, sorted_ids, ntpp,
                      capacity, row_weight, a1, a1_scale);
  if (fp8)
    return launch_pdl(gather_kernel<kGatherFp8>, blocks, 256, 0, stream, xb, H, topk, nflat, sorted_ids, ntpp,
                      capacity, row_weight, a1, a1_scale);
  return launch_pdl(gather_kernel<kGatherBf16>, blocks, 256, 0, stream, xb, H, topk, nflat, sorted_ids, ntpp,
                    capacity, row_weight, a1, a1_scale);
}

// ----------------------------------------------------------------------------
// Quantise x once per token (T rows, not T * topk): E4M3 codes into xq [T, H];
// each (token, K block) scale is written to the sorted rows of the token's
// topk assignments (pos_of_flat, the inverse of sorted_token_ids) -- fp32
// a1_scale_t [H/128, capacity] (FP8, rule of vLLM PR #64760 analysis §1.2)
// or E8M0 bytes in the SF-atom layout of [capacity, H] (MXFP8).  The GEMM1
// producer gathers the code rows with TMA tile::gather4, so the sorted copy
// of x never reaches HBM.  row_weight (top-1 only): the row is first
// bf16(fp32(x) * w).
// ----------------------------------------------------------------------------
template <bool MX>
__global__ void __launch_bounds__(256) quantize_x_kernel(const __nv_bfloat16* x, int T, int H, int topk,
                                                         const int32_t* pos_of_flat, int capacity,
                                                         const float* row_weight, uint8_t* xq, void* scales,
                                                         int split) {
  pdl_launch_dependents();
  pdl_wait();
  const int vecs = H / 8;
  const int chunks = (vecs + blockDim.x - 1) / blockDim.x;  // 256-vector chunks of a row
  // split = 1: a block takes whole rows; split = chunks (few rows): one chunk of a row
  const long long items = static_cast<long long>(T) * split;
  for (long long item = blockIdx.x; item < items; item += gridDim.x) {
    const int t = static_cast<int>(item / split);
    const int c0 = static_cast<int>(item - static_cast<long long>(t) * split);
    const float rw = row_weight ? (*(row_weight + static_cast<size_t>(t) * topk)) : 1.0f;
    const __nv_bfloat16* src = x + static_cast<size_t>(t) * H;
    for (int it = c0; it < chunks; it += split) {
      const int v = it * blockDim.x + threadIdx.x;  // uniform trip count: shuffles see full warps
      const bool in = v < vecs;
      uint4 u = make_uint4(0, 0, 0, 0);
      if (in) u = (*(reinterpret_cast<const uint4*>(src) + v));
      float f[8];
      unpack8(u, f);
      if (row_weight) {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = bf16_round(f[i] * rw);
      }
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
      for (int off = (MX ? 2 : 8); off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const float scale = act_scale_from_amax(amax);
      const float inv = pow2_recip(scale);
      uint2 q;
      q.x = static_cast<uint32_t>(f32x2_to_e4m3x2(f[0] * inv, f[1] * inv)) |
            (static_cast<uint32_t>(f32x2_to_e4m3x2(f[2] * inv, f[3] * inv)) << 16);
      q.y = static_cast<uint32_t>(f32x2_to_e4m3x2(f[4] * inv, f[5] * inv)) |
            (static_cast<uint32_t>(f32x2_to_e4m3x2(f[6] * inv, f[7] * inv)) << 16);
      if (in) {
        reinterpret_cast<uint2*>(xq + static_cast<size_t>(t) * H)[v] = q;
        if ((v & (MX ? 3 : 15)) == 0) {
          for (int j = 0; j < topk; ++j) {
            const int r = (*(pos_of_flat + static_cast<size_t>(t) * topk + j));
            if (r < 0) continue;  // invalid expert id: the assignment has no row
            if constexpr (MX)
              static_cast<uint8_t*>(scales)[sf_atom_offset(r, v * 8, H)] = e8m0_of_pow2(scale);
            else
              static_cast<float*>(scales)[static_cast<size_t>(v >> 4) * capacity + r] = scale;
          }
        }
      }
    }
  }
}

// bf16 rows scaled by the router weight (top-1): out[t] = bf16(fp32(x[t]) * w[t])
__global__ void __launch_bounds__(256) scale_rows_kernel(const __nv_bfloat16* x, int T, int H, int topk,
                                                         const float* row_weight, __nv_bfloat16* out) {
  pdl_launch_dependents();
  pdl_wait();
  const int vecs = H / 8;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const float rw = (*(row_weight + static_cast<size_t>(t) * topk));
    for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
      float f[8];
      unpack8((*(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H) + v)), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] *= rw;
      reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H)[v] = pack8(f);
    }
  }
}

// ----------------------------------------------------------------------------
// Sorted copy of quantised rows: a1[pos_of_flat[f]] = xq[f / topk] (E4M3 bytes)
// for every assignment f that has a row.  With the per-token quantiser in
// front, x is read and quantised once per token instead of once per
// assignment; this copy then reads the L2-resident codes.  One warp per row:
// each lane issues its 16-byte loads of a 4 KB piece of the row before any
// store, and the 64 warps an SM holds keep that many rows in flight.
// Padding rows are never stored (GEMM1 reads them; their outputs are dropped).
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) copy_rows_kernel(const uint8_t* xq, int H, int topk, int nflat,
                                                        const int32_t* pos_of_flat, uint8_t* a1) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int kPer = 8;  // 16-byte vectors per lane in flight
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int vecs = H / 16;
  for (int f = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); f < nflat; f += warps) {
    const int row = (*(pos_of_flat + f));
    if (row < 0) continue;  // an invalid expert id (or another rank's expert): no row
    const uint4* src = reinterpret_cast<const uint4*>(xq + static_cast<size_t>(f / topk) * H);
    uint4* dst = reinterpret_cast<uint4*>(a1 + static_cast<size_t>(row) * H);
    for (int base = 0; base < vecs; base += kPer * 32) {
      uint4 v[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int k = base + i * 32 + lane;
        if (k < vecs) v[i] = (*(src + k));
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int k = base + i * 32 + lane;
        if (k < vecs) dst[k] = v[i];
      }
    }
  }
}

cudaError_t launch_copy_rows(const void* xq, int H, int topk, int nflat, const int32_t* pos_of_flat, void* a1,
                             cudaStream_t stream) {
  if (nflat == 0) return cudaSuccess;
  if (pos_of_flat == nullptr) return cudaErrorInvalidValue;
  const int want = (nflat + 7) / 8;  // eight warps (rows) per block
  const int blocks = want < 148 * 8 ? want : 148 * 8;
  return launch_pdl(copy_rows_kernel, blocks, 256, 0, stream, static_cast<const uint8_t*>(xq), H, topk, nflat,
                    pos_of_flat, static_cast<uint8_t*>(a1));
}

cudaError_t launch_prepare_x(const void* x, int T, int H, int topk, bool fp8, bool mx, const int32_t* pos_of_flat,
                             int capacity, const float* row_weight, void* xq, void* scales, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  // whole rows per block when the rows alone fill the grid; else a block per 256-vector chunk of a row
  const int chunks = (H / 8 + 255) / 256;
  const int split = T >= 148 * 8 ? 1 : chunks;
  const long long items = static_cast<long long>(T) * split;
  const int blocks = items < 148 * 8 ? static_cast<int>(items) : 148 * 8;
  const int row_blocks = T < 148 * 8 ? T : 148 * 8;  // scale_rows_kernel: one row per block
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (mx)
    return launch_pdl(quantize_x_kernel<true>, blocks, 256, 0, stream, xb, T, H, topk, pos_of_flat, capacity,
                      row_weight, static_cast<uint8_t*>(xq), scales, split);
  if (fp8)
    return launch_pdl(quantize_x_kernel<false>, blocks, 256, 0, stream, xb, T, H, topk, pos_of_flat, capacity,
                      row_weight, static_cast<uint8_t*>(xq), scales, split);
  if (row_weight)
    return launch_pdl(scale_rows_kernel, row_blocks, 256, 0, stream, xb, T, H, topk, row_weight,
                      static_cast<__nv_bfloat16*>(xq));
  return cudaSuccess;
}

// ----------------------------------------------------------------------------
// combine ("Hosting von Qwen auf Blackwell", "MoE Dispatch - Combine": the
// weighted accumulation; the weights were applied in the GEMM2 epilogue):
// out[t, :] = bf16(sum_j y[t*topk + j, :]) in fp32, j ascending.  kMasked
// (expert parallelism, "Experten-Parallel": the local accumulation before the
// all-reduce): only the assignments with a row on this rank, pos_of_flat >= 0;
// a token without one gets zeros.
// ----------------------------------------------------------------------------
template <bool kMasked>
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* y, int T, int topk, int H,
                                                      const int32_t* pos_of_flat, __nv_bfloat16* out) {
  pdl_launch_dependents();
  pdl_wait();
  const int vecs = H / 8;
  const long long total = static_cast<long long>(T) * vecs;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = i / vecs;
    const int v = static_cast<int>(i - t * vecs);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const uint4* src = reinterpret_cast<const uint4*>(y + static_cast<size_t>(t) * topk * H) + v;
    for (int j = 0; j < topk; ++j) {
      if (kMasked && (*(pos_of_flat + static_cast<size_t>(t) * topk + j)) < 0) continue;  // never written
      float f[8];
      unpack8((*(src + static_cast<size_t>(j) * vecs)), f);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] += f[k];
    }
    reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H)[v] = pack8(acc);
  }
}

cudaError_t launch_combine(const void* y, int T, int topk, int H, const int32_t* pos_of_flat, void* out,
                           cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const long long total = static_cast<long long>(T) * (H / 8);
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  const auto* yb = static_cast<const __nv_bfloat16*>(y);
  auto* ob = static_cast<__nv_bfloat16*>(out);
  if (pos_of_flat)
    return launch_pdl(combine_kernel<true>, static_cast<int>(blocks), 256, 0, stream, yb, T, topk, H, pos_of_flat,
                      ob);
  return launch_pdl(combine_kernel<false>, static_cast<int>(blocks), 256, 0, stream, yb, T, topk, H, pos_of_flat, ob);
}

// ----------------------------------------------------------------------------
// weight preparation: one CTA per 128x128 block; thread = half a row (64
// elements).  scale = max(blockmax, 1e-10) / 448 and code = e4m3(w / scale),
// both divisions correctly rounded in fp32.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_weights_kernel(const __nv_bfloat16* w, int rows,
                                                               int cols, uint8_t* codes,
                                                               float* scales) {
  __shared__ float warp_max[8];
  pdl_launch_dependents();
  pdl_wait();
  const int nbc = cols / 128, nbr = rows / 128;
  const long long blk = blockIdx.x;
  const long long b = blk / (static_cast<long long>(nbr) * nbc);
  const int rem = static_cast<int>(blk - b * nbr * nbc);
  const int br = rem / nbc, bc = rem - br * nbc;
  const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
  const size_t row_off = (static_cast<size_t>(b) * rows + static_cast<size_t>(br) * 128 + r) * cols +
                         static_cast<size_t>(bc) * 128 + half * 64;
  const uint4* src = reinterpret_cast<const uint4*>(w + row_off);
  float f[64];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float t[8];
    unpack8((*(src + i)), t);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      f[8 * i + k] = t[k];
      amax = fmaxf(amax, fabsf(t[k]));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  float bmax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) bmax = fmaxf(bmax, warp_max[i]);
  const float scale = __fdiv_rn(fmaxf(bmax, 1e-10f), 448.0f);
  uint4* dst = reinterpret_cast<uint4*>(codes + row_off);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t wds[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = 16 * i + 4 * j;
      wds[j] = static_cast<uint32_t>(f32x2_to_e4m3x2(__fdiv_rn(f[k], scale), __fdiv_rn(f[k + 1], scale))) |
               (static_cast<uint32_t>(f32x2_to_e4m3x2(__fdiv_rn(f[k + 2], scale), __fdiv_rn(f[k + 3], scale)))
                << 16);
    }
    dst[i] = make_uint4(wds[0], wds[1], wds[2], wds[3]);
  }
  if (threadIdx.x == 0) scales[blk] = scale;
}

cudaError_t launch_quantize_weights(const void* w, long long batches, int rows, int cols, uint8_t* codes,
                                    float* scales, cudaStream_t stream) {
  const long long blocks = batches * (rows / 128) * (cols / 128);
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  return launch_pdl(quantize_weights_kernel, static_cast<unsigned>(blocks), 256, 0, stream,
                    static_cast<const __nv_bfloat16*>(w), rows, cols, codes, scales);
}

// ----------------------------------------------------------------------------
// MXFP8 weight quantisation: one CTA per 128x128 block, thread = (row, 64
// columns) = two 32-column groups.  scale = pow2 ceiling of fp32(max(amax,
// 1e-10)) * fp32(1/448); code = e4m3(w * 2^-e) (exact scaling, RNE,
// saturating); the E8M0 bytes go to the SF-atom layout.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_weights_mx_kernel(const __nv_bfloat16* w, int rows, int cols,
                                                                  uint8_t* codes, uint8_t* sf) {
  pdl_launch_dependents();
  pdl_wait();
  const int nbc = cols / 128, nbr = rows / 128;
  const long long blk = blockIdx.x;
  const long long b = blk / (static_cast<long long>(nbr) * nbc);
  const int rem = static_cast<int>(blk - b * nbr * nbc);
  const int br = rem / nbc, bc = rem - br * nbc;
  const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
  const long long grow = b * rows + static_cast<long long>(br) * 128 + r;  // row in the batch of matrices
  const int col0 = bc * 128 + half * 64;
  const size_t row_off = static_cast<size_t>(grow) * cols + col0;
  const uint4* src = reinterpret_cast<const uint4*>(w + row_off);
  uint4* dst = reinterpret_cast<uint4*>(codes + row_off);
  uint8_t e8[2];
#pragma unroll
  for (int grp = 0; grp < 2; ++grp) {
    float f[32];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float t[8];
      unpack8((*(src + 4 * grp + i)), t);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        f[8 * i + k] = t[k];
        amax = fmaxf(amax, fabsf(t[k]));
      }
    }
    const float scale = act_scale_from_amax(amax);
    const float inv = pow2_recip(scale);
    uint32_t wds[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      wds[i] = static_cast<uint32_t>(f32x2_to_e4m3x2(f[4 * i] * inv, f[4 * i + 1] * inv)) |
               (static_cast<uint32_t>(f32x2_to_e4m3x2(f[4 * i + 2] * inv, f[4 * i + 3] * inv)) << 16);
    dst[2 * grp] = make_uint4(wds[0], wds[1], wds[2], wds[3]);
    dst[2 * grp + 1] = make_uint4(wds[4], wds[5], wds[6], wds[7]);
    e8[grp] = e8m0_of_pow2(scale);
  }
  // the thread's two groups are adjacent bytes of one SF-atom row
  *reinterpret_cast<uint16_t*>(sf + sf_atom_offset(grow, col0, cols)) =
      static_cast<uint16_t>(e8[0] | (static_cast<uint16_t>(e8[1]) << 8));
}

cudaError_t launch_quantize_weights_mx(const void* w, long long batches, int rows, int cols, uint8_t* codes,
                                       uint8_t* sf, cudaStream_t stream) {
  const long long blocks = batches * (rows / 128) * (cols / 128);
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  return launch_pdl(quantize_weights_mx_kernel, static_cast<unsigned>(blocks), 256, 0, stream,
                    static_cast<const __nv_bfloat16*>(w), rows, cols, codes, sf);
}

}  // namespace moe
