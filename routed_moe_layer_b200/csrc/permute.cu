// Token -> expert permutation (xxqk.cn vLLM-Omni article, "MoE 实现的源码级要点":
// tokens are reordered so that each expert's rows are contiguous before the
// grouped expert GEMMs).
//
// A stable counting sort keyed by expert: row(t, j) = offset[e] + #{t' < t :
// e in ids[t']} with e = ids[t, j] (a token never holds an expert twice), so
// rows are ordered by expert, then token -- unique and deterministic.
//   1. count:   per 32-token warp, one bit per token in a per-expert mask;
//               block histogram = popcounts of the masks.
//   2. scan:    one CTA turns the block histograms into per-block row bases
//               and per-expert offsets (+ the prefix of 128-row GEMM tiles).
//   3. scatter: rank inside the warp = popcount of the lower lanes' bits;
//               also the token-major slot position of every row.
//   4. gather:  xp[row] = x[tok_of[row]], walking tokens in order so that each
//               token row is read once (skipped when x is not given).
// Up to PERMUTE_SMALL_T tokens, steps 1-4 run in one launch: every CTA of a
// small grid computes steps 1-3 for all tokens in shared memory (one token
// per thread; the same deterministic result in each CTA, so no CTA waits for
// another), CTA 0 writes the offsets, and each CTA writes the rows of, and
// gathers, its own share of the tokens.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace rmoe {

namespace {

constexpr int PT = PERMUTE_TOK;      // tokens per block (8 warps)
constexpr int PW = PERMUTE_TOK / 32; // warps per block
constexpr int MAXE = 128;
constexpr int MAX_TOPK_PERMUTE = 16;

__device__ __forceinline__ void build_masks(const int32_t* __restrict__ ids, int T, int E,
                                            int top_k, const uint8_t* __restrict__ tmask,
                                            uint32_t (*masks)[MAXE], int* status) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < PW * MAXE; i += PT) (&masks[0][0])[i] = 0u;
  __syncthreads();
  const int t = blockIdx.x * PT + tid;
  if (t < T && (!tmask || tmask[t] != 0)) {  // padding tokens take no rows
    for (int j = 0; j < top_k; ++j) {
      const int e = ids[(size_t)t * top_k + j];
      if (e >= 0 && e < E)
        atomicOr(&masks[warp][e], 1u << lane);
      else
        report_error(status, MOE_ERR_DEVICE_INDEX, 1);
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(PT)
    permute_count_kernel(const int32_t* __restrict__ ids, int T, int E, int top_k,
                         const uint8_t* __restrict__ tmask, int* __restrict__ blk_hist,
                         int* status) {
  __shared__ uint32_t masks[PW][MAXE];
  pdl_launch_dependents();
  pdl_wait();
  build_masks(ids, T, E, top_k, tmask, masks, status);
  for (int e = threadIdx.x; e < E; e += PT) {
    int cnt = 0;
#pragma unroll
    for (int w = 0; w < PW; ++w) cnt += __popc(masks[w][e]);
    blk_hist[(size_t)blockIdx.x * E + e] = cnt;
  }
}

// Warp 0 of a CTA: exclusive prefixes over experts of the row counts tot[e]
// and of their MTILE-row tiles, into excl_rows / excl_tiles [E+1] (shared).
__device__ __forceinline__ void scan_experts_warp(const int* tot_of, int E, int* excl_rows,
                                                  int* excl_tiles) {
  const int lane = threadIdx.x & 31;
  int loc_rows[MAXE / 32], loc_tiles[MAXE / 32];
  int sr = 0, st = 0;
#pragma unroll
  for (int q = 0; q < MAXE / 32; ++q) {
    const int ee = lane * (MAXE / 32) + q;
    const int tot = ee < E ? tot_of[ee] : 0;
    loc_rows[q] = tot;
    loc_tiles[q] = (tot + MTILE - 1) / MTILE;
    sr += loc_rows[q];
    st += loc_tiles[q];
  }
  int ir = sr, it = st;  // inclusive warp scan of the per-lane sums
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, ir, off);
    const int b = __shfl_up_sync(0xffffffffu, it, off);
    if (lane >= off) {
      ir += a;
      it += b;
    }
  }
  int run_r = ir - sr, run_t = it - st;
#pragma unroll
  for (int q = 0; q < MAXE / 32; ++q) {
    const int ee = lane * (MAXE / 32) + q;
    if (ee < E) {
      excl_rows[ee] = run_r;
      excl_tiles[ee] = run_t;
    }
    run_r += loc_rows[q];
    run_t += loc_tiles[q];
  }
  if (lane == 31) {
    excl_rows[E] = ir;
    excl_tiles[E] = it;
  }
}

// Writes the per-expert row offsets and tile prefixes ([E+1], plus group E+1
// when extra_rows > 0) from the shared exclusive prefixes; threads 0..E.
__device__ __forceinline__ void write_offsets(const int* excl_rows, const int* excl_tiles, int E,
                                              int extra_rows, int* expert_offsets,
                                              int* mtile_start) {
  const int tid = threadIdx.x;
  if (tid <= E) {
    expert_offsets[tid] = excl_rows[tid];
    if (mtile_start) mtile_start[tid] = excl_tiles[tid];
  }
  if (tid == 0 && extra_rows > 0) {  // one more group after the experts
    expert_offsets[E + 1] = excl_rows[E] + extra_rows;
    if (mtile_start) mtile_start[E + 1] = excl_tiles[E] + (extra_rows + MTILE - 1) / MTILE;
  }
}

// One CTA of 1024 threads: expert e = tid % E, chunk ch = tid / E of the blocks.
__global__ void __launch_bounds__(1024)
    permute_scan_kernel(int* __restrict__ blk_hist, int nblk, int E, int extra_rows,
                        int* __restrict__ expert_offsets, int* __restrict__ mtile_start) {
  __shared__ int part[1024];
  __shared__ int tot[MAXE];
  __shared__ int excl_rows[MAXE + 1];
  __shared__ int excl_tiles[MAXE + 1];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x;
  const int C = 1024 / E;
  const int e = tid % E, ch = tid / E;
  const bool active = ch < C;
  int b0 = 0, b1 = 0;
  if (active) {
    b0 = (int)((long long)ch * nblk / C);
    b1 = (int)((long long)(ch + 1) * nblk / C);
    int s = 0;
    for (int b = b0; b < b1; ++b) s += blk_hist[(size_t)b * E + e];
    part[ch * E + e] = s;
  }
  __syncthreads();
  if (tid < E) {  // per-expert total; chunk sums become exclusive prefixes over chunks
    int run = 0;
    for (int c = 0; c < C; ++c) {
      const int v = part[c * E + tid];
      part[c * E + tid] = run;
      run += v;
    }
    tot[tid] = run;
  }
  __syncthreads();
  if (tid < 32) scan_experts_warp(tot, E, excl_rows, excl_tiles);
  __syncthreads();
  write_offsets(excl_rows, excl_tiles, E, extra_rows, expert_offsets, mtile_start);
  if (active) {
    int run = excl_rows[e] + part[ch * E + e];
    for (int b = b0; b < b1; ++b) {
      const size_t i = (size_t)b * E + e;
      const int v = blk_hist[i];
      blk_hist[i] = run;  // base row of expert e inside block b
      run += v;
    }
  }
}

// T <= PERMUTE_SMALL_T: count, scan and scatter with one token per thread
// (1024 threads); the same rows as the three-kernel path.  Every CTA computes
// the whole permutation; CTA 0 writes the offsets; CTA b writes the rows of
// tokens [b*per, (b+1)*per) and, when x is given, gathers them into xp.
constexpr int SMALL_PER_MAX = 64;  // tokens per CTA
__global__ void __launch_bounds__(1024)
    permute_small_kernel(const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T,
                         int E, int top_k, int extra_rows, int* __restrict__ expert_offsets,
                         int* __restrict__ mtile_start, int* __restrict__ row_of,
                         int* __restrict__ tok_of, float* __restrict__ w_of,
                         int* __restrict__ pos_of, int slot_stride,
                         const uint8_t* __restrict__ tmask, int* status,
                         const __nv_bfloat16* __restrict__ x, int H, int per,
                         __nv_bfloat16* __restrict__ xp) {
  __shared__ uint32_t masks[32][MAXE];
  __shared__ int wbase[32][MAXE];
  __shared__ int tot[MAXE];
  __shared__ int excl_rows[MAXE + 1];
  __shared__ int excl_tiles[MAXE + 1];
  __shared__ int rows_sm[SMALL_PER_MAX][MAX_TOPK_PERMUTE];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < 32 * MAXE; i += 1024) (&masks[0][0])[i] = 0u;
  __syncthreads();
  const int t = tid;
  const bool real = t < T && (!tmask || tmask[t] != 0);  // padding tokens take no rows
  int my_e[MAX_TOPK_PERMUTE];
  float my_w[MAX_TOPK_PERMUTE];  // loaded with the ids, off the scatter's critical path
#pragma unroll
  for (int j = 0; j < MAX_TOPK_PERMUTE; ++j) {
    my_e[j] = -1;
    my_w[j] = 1.0f;
    if (real && j < top_k) {
      if (topk_w) my_w[j] = topk_w[(size_t)t * top_k + j];
      const int e = ids[(size_t)t * top_k + j];
      if (e >= 0 && e < E) {
        my_e[j] = e;
        atomicOr(&masks[warp][e], 1u << lane);
      } else if (blockIdx.x == 0) {
        report_error(status, MOE_ERR_DEVICE_INDEX, 1);
      }
    }
  }
  __syncthreads();
  if (tid < E) {  // rows of expert e before each warp, and in total
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      wbase[w][tid] = run;
      run += __popc(masks[w][tid]);
    }
    tot[tid] = run;
  }
  __syncthreads();
  if (tid < 32) scan_experts_warp(tot, E, excl_rows, excl_tiles);
  __syncthreads();
  if (blockIdx.x == 0) write_offsets(excl_rows, excl_tiles, E, extra_rows, expert_offsets, mtile_start);
  const int t_lo = blockIdx.x * per, t_hi = min(T, t_lo + per);
  if (t >= t_lo && t < t_hi) {
    const uint32_t lower = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < MAX_TOPK_PERMUTE; ++j) {
      if (j >= top_k) break;
      const size_t tj = (size_t)t * top_k + j;
      const int e = my_e[j];
      int row = -1;
      if (e >= 0) {
        row = excl_rows[e] + wbase[warp][e] + __popc(masks[warp][e] & lower);
        tok_of[row] = t;
        if (w_of) w_of[row] = my_w[j];
        if (pos_of) pos_of[row] = t * slot_stride + j;
      }
      row_of[tj] = row;
      rows_sm[t - t_lo][j] = row;
    }
  }
  if (!x || !xp) return;
  __syncthreads();
  // gather: this CTA's tokens, 32-byte pieces of a row, every piece to each of
  // the token's rows (x read once)
  const int pieces = H / 16;
  const int n = (t_hi - t_lo) * pieces;
  for (int c = tid; c < n; c += 1024) {
    const int tl = c / pieces, pc = c - tl * pieces;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(t_lo + tl) * H + 16 * pc);
    const uint4 a = src[0], b = src[1];
    const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    for (int j = 0; j < top_k; ++j) {
      const int r = rows_sm[tl][j];
      if (r >= 0) st_global_v8(xp + (size_t)r * H + 16 * pc, v);
    }
  }
}

__global__ void __launch_bounds__(PT)
    permute_scatter_kernel(const int32_t* __restrict__ ids, const float* __restrict__ topk_w,
                           int T, int E, int top_k, const int* __restrict__ blk_base,
                           int* __restrict__ row_of, int* __restrict__ tok_of,
                           float* __restrict__ w_of, int* __restrict__ pos_of, int slot_stride,
                           const uint8_t* __restrict__ tmask, int* status) {
  __shared__ uint32_t masks[PW][MAXE];
  __shared__ int wbase[PW][MAXE];
  pdl_launch_dependents();
  pdl_wait();
  build_masks(ids, T, E, top_k, tmask, masks, status);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < E; e += PT) {
    int run = blk_base[(size_t)blockIdx.x * E + e];
#pragma unroll
    for (int w = 0; w < PW; ++w) {
      wbase[w][e] = run;
      run += __popc(masks[w][e]);
    }
  }
  __syncthreads();
  const int t = blockIdx.x * PT + tid;
  if (t >= T) return;
  const bool pad = tmask && tmask[t] == 0;
  const uint32_t lower = (1u << lane) - 1u;
  for (int j = 0; j < top_k; ++j) {
    const size_t tj = (size_t)t * top_k + j;
    const int e = pad ? -1 : ids[tj];
    if (e < 0 || e >= E) {
      row_of[tj] = -1;
      continue;
    }
    const int row = wbase[warp][e] + __popc(masks[warp][e] & lower);
    row_of[tj] = row;
    tok_of[row] = t;
    if (w_of) w_of[row] = topk_w ? topk_w[tj] : 1.0f;
    if (pos_of) pos_of[row] = t * slot_stride + j;
  }
}

// One warp per token (small batches: several): x[t] is read once (1 KB per
// warp step: 32 bytes per lane) and written to the token's top_k rows with
// full-sector stores; row_of gives the rows (-1: skipped id), fetched once.
__global__ void __launch_bounds__(256)
    gather_tokens_kernel(const __nv_bfloat16* __restrict__ x, const int* __restrict__ row_of,
                         int T, int H, int top_k, int parts, __nv_bfloat16* __restrict__ xp) {
  __shared__ int rows_sm[8][MAX_TOPK_PERMUTE];  // each warp's current token's rows
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int chunks = H / 16;  // 32-byte pieces of a row (H is a multiple of 64)
  int* rows = rows_sm[wib];
  // `parts` warps share a token (small batches), each taking every parts-th
  // 1 KB column block of the row
  for (int wt = blockIdx.x * (blockDim.x >> 5) + wib; wt < T * parts; wt += warps) {
    const int t = wt / parts, part = wt - t * parts;
    __syncwarp();  // the previous token's rows have been used
    if (lane < top_k) rows[lane] = row_of[(size_t)t * top_k + lane];
    __syncwarp();
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    for (int c = lane + 32 * part; c < chunks; c += 32 * parts) {
      const uint4 a = src[2 * c], b = src[2 * c + 1];
      const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      for (int j = 0; j < top_k; ++j) {
        const int r = rows[j];
        if (r >= 0) st_global_v8(xp + (size_t)r * H + 16 * c, v);
      }
    }
  }
}

cudaError_t launch_gather(const void* x, int T, int H, int top_k, const PermuteOut& o,
                          cudaStream_t stream) {
  if (o.xp && x) {
    // warps per token: enough warps to fill the GPU twice over, at most one
    // per 1 KB column block of a row
    const int cap = num_sms() * 8;  // blocks of 8 warps
    int parts = (2 * cap * 8) / (T > 0 ? T : 1);
    const int max_parts = H / 512;
    if (parts > max_parts) parts = max_parts;
    if (parts < 1) parts = 1;
    long long grid = ((long long)T * parts + 7) / 8;
    if (grid > cap) grid = cap;
    const cudaError_t err = launch_chained(
        gather_tokens_kernel, dim3((unsigned)grid), dim3(256), 0, stream,
        static_cast<const __nv_bfloat16*>(x), (const int*)o.row_of, T, H, top_k, parts,
        static_cast<__nv_bfloat16*>(o.xp));
    if (err != cudaSuccess) return err;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_permute(const int32_t* topk_ids, const float* topk_w, const void* x, int T,
                           int H, int E, int top_k, const PermuteOut& o, cudaStream_t stream) {
  cudaError_t err;
  if (T <= PERMUTE_SMALL_T) {
    // with a gather: about 8 tokens per CTA (at most one CTA per SM); without: one CTA
    const bool gather = x && o.xp;
    int grid = gather ? std::min(num_sms(), (T + 7) / 8) : 1;
    if (grid < 1) grid = 1;
    int per = (T + grid - 1) / grid;
    if (per > SMALL_PER_MAX) {
      per = SMALL_PER_MAX;
      grid = (T + per - 1) / per;
    }
    err = launch_chained(permute_small_kernel, dim3(grid), dim3(1024), 0, stream, topk_ids, topk_w,
                         T, E, top_k, o.extra_rows, o.expert_offsets, o.mtile_start, o.row_of,
                         o.tok_of, o.w_of, o.pos_of, o.slot_stride, o.mask, o.status,
                         static_cast<const __nv_bfloat16*>(gather ? x : nullptr), H, per,
                         static_cast<__nv_bfloat16*>(gather ? o.xp : nullptr));
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
  }
  const int nblk = (T + PT - 1) / PT;
  err = launch_chained(permute_count_kernel, dim3(nblk), dim3(PT), 0, stream, topk_ids, T, E,
                       top_k, o.mask, o.blk_hist, o.status);
  if (err != cudaSuccess) return err;
  err = launch_chained(permute_scan_kernel, dim3(1), dim3(1024), 0, stream, o.blk_hist, nblk, E,
                       o.extra_rows, o.expert_offsets, o.mtile_start);
  if (err != cudaSuccess) return err;
  err = launch_chained(permute_scatter_kernel, dim3(nblk), dim3(PT), 0, stream, topk_ids, topk_w,
                       T, E, top_k, (const int*)o.blk_hist, o.row_of, o.tok_of, o.w_of, o.pos_of,
                       o.slot_stride, o.mask, o.status);
  if (err != cudaSuccess) return err;
  return launch_gather(x, T, H, top_k, o, stream);
}

}  // namespace rmoe
