// Kernels of the expert-parallel form of the block: experts split across
// ranks, each rank routing its own tokens and sending every (token, slot) row
// to the rank that holds its expert (an all-to-all each way between the two
// grouped GEMMs).  The block's arithmetic is unchanged (sglang PR #32341
// report, LingBotVideoSparseMoeBlock.forward: router -> grouped experts with
// the router weight on the output -> restore -> + shared expert); only where
// the rows are computed changes.
//   rows_expert_ids  expert id of every row of an expert-sorted row list
//   tile_prefix      prefix of 256-row tiles per group (the pair GEMM's schedule)
//   combine_rows     the restore with the routed rows addressed through row_of:
//                    out[t] = bf16( sum_j y[row_of[t,j]] + shared[t] + residual[t] ),
//                    fp32, slots in order, then shared, then residual -- the
//                    same sums in the same order as the block's own restore
#include "common.cuh"
#include "kernels.h"

namespace rmoe {

namespace {

__global__ void __launch_bounds__(256)
    rows_expert_ids_kernel(const int* __restrict__ offsets, int E, int R, int* __restrict__ ids) {
  pdl_launch_dependents();
  pdl_wait();
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < R; r += gridDim.x * blockDim.x) {
    int lo = 0, hi = E;  // largest e with offsets[e] <= r + offsets[0]
    const int row = r + offsets[0];
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (offsets[mid] <= row)
        lo = mid;
      else
        hi = mid;
    }
    ids[r] = lo;
  }
}

__global__ void __launch_bounds__(32)
    tile_prefix_kernel(const int* __restrict__ offsets, int groups, int* __restrict__ tiles) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int PER = 5;  // groups per lane (up to 160)
  const int lane = threadIdx.x;
  int loc[PER], sum = 0;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int g = lane * PER + q;
    loc[q] = g < groups ? (offsets[g + 1] - offsets[g] + MTILE - 1) / MTILE : 0;
    sum += loc[q];
  }
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  int run = incl - sum;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int g = lane * PER + q;
    if (g <= groups) tiles[g] = run;
    run += loc[q];
  }
}

// One warp per token (small batches: up to H/256 warps, each on every
// parts-th 512-byte column block); 16-byte loads and stores.
__global__ void __launch_bounds__(256)
    combine_rows_kernel(const __nv_bfloat16* __restrict__ y, int R, const int* __restrict__ row_of,
                        int top_k, int T, int H, int parts,
                        const __nv_bfloat16* __restrict__ shared,
                        const __nv_bfloat16* __restrict__ residual,
                        __nv_bfloat16* __restrict__ out) {
  __shared__ int rows_sm[8][16];
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int hv = H / 8;  // 16-byte vectors per row
  int* rows = rows_sm[wib];
  for (int wt = blockIdx.x * (blockDim.x >> 5) + wib; wt < T * parts; wt += warps) {
    const int t = wt / parts, part = wt - t * parts;
    __syncwarp();
    if (lane < top_k) rows[lane] = row_of[(size_t)t * top_k + lane];
    __syncwarp();
    for (int c = lane + 32 * part; c < hv; c += 32 * parts) {
      float s[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i] = 0.f;
      auto add = [&](const uint4& v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          s[2 * i] += bf16_lo(w[i]);
          s[2 * i + 1] += bf16_hi(w[i]);
        }
      };
      for (int j = 0; j < top_k; ++j) {  // a rejected id (or a row outside y) adds 0
        const int r = rows[j];
        add(r >= 0 && r < R ? reinterpret_cast<const uint4*>(y + (size_t)r * H)[c]
                            : make_uint4(0, 0, 0, 0));
      }
      if (shared) add(reinterpret_cast<const uint4*>(shared + (size_t)t * H)[c]);
      if (residual) add(reinterpret_cast<const uint4*>(residual + (size_t)t * H)[c]);
      reinterpret_cast<uint4*>(out + (size_t)t * H)[c] =
          make_uint4(pack_bf16x2(s[0], s[1]), pack_bf16x2(s[2], s[3]), pack_bf16x2(s[4], s[5]),
                     pack_bf16x2(s[6], s[7]));
    }
  }
}

}  // namespace

cudaError_t launch_rows_expert_ids(const int* offsets, int E, int R, int* ids,
                                   cudaStream_t stream) {
  if (R <= 0) return cudaSuccess;
  long long grid = ((long long)R + 255) / 256;
  if (grid > num_sms() * 8) grid = num_sms() * 8;
  return launch_chained(rows_expert_ids_kernel, dim3((unsigned)grid), dim3(256), 0, stream,
                        offsets, E, R, ids);
}

cudaError_t launch_tile_prefix(const int* offsets, int groups, int* tiles, cudaStream_t stream) {
  if (groups < 1 || groups > 159) return cudaErrorInvalidValue;
  return launch_chained(tile_prefix_kernel, dim3(1), dim3(32), 0, stream, offsets, groups, tiles);
}

cudaError_t launch_combine_rows(const void* y, int R, const int* row_of, int top_k, int T, int H,
                                const void* shared, const void* residual, void* out,
                                cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  if (top_k > 16) return cudaErrorInvalidValue;
  const int cap = num_sms() * 8;  // blocks of 8 warps
  int parts = (2 * cap * 8) / T;
  const int max_parts = H / 256;
  if (parts > max_parts) parts = max_parts;
  if (parts < 1) parts = 1;
  long long grid = ((long long)T * parts + 7) / 8;
  if (grid > cap) grid = cap;
  return launch_chained(combine_rows_kernel, dim3((unsigned)grid), dim3(256), 0, stream,
                        static_cast<const __nv_bfloat16*>(y), R, row_of, top_k, T, H, parts,
                        static_cast<const __nv_bfloat16*>(shared),
                        static_cast<const __nv_bfloat16*>(residual),
                        static_cast<__nv_bfloat16*>(out));
}

}  // namespace rmoe
