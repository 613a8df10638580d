// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

namespace rmoe {

// A kernel's dynamic shared-memory limit is an attribute of the kernel in one
// device's context, so it is set once per device: `done` is a per-call-site
// table indexed by device ordinal (devices beyond it set it on every launch).
constexpr int MAX_DEVICES = 64;
template <typename... KArgs>
cudaError_t set_smem_limit_per_device(void (*k)(KArgs...), int bytes,
                                      std::atomic<int> (&done)[MAX_DEVICES]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < MAX_DEVICES && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < MAX_DEVICES) done[dev].store(1, std::memory_order_release);
  return e;
}

// Launches kernel k chained to the previous work of the stream (programmatic
// stream serialisation; the kernel itself waits with pdl_wait before reading
// what its predecessors wrote).
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t stream, Args&&... args) {
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
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}

struct RouterParams {
  int T, H, E, top_k, n_group, topk_group, norm_topk_prob;
  float rsf;
  int clear_status;  // 1: the router's first kernel clears the status word
  const uint8_t* mask = nullptr;  // [T] or null: 0 = padding token (ids -1, weights 0)
  int* zero = nullptr;  // [zero_n] ints the router's first kernel sets to 0 (counters of
  int zero_n = 0;       //   later kernels of the same forward), or null
};

// Router on the tensor cores: scratch holds the 3-term bf16 split of Wr and the
// fp32 partial logits of the K chunks (router_scratch_bytes).
int router_splits(int H);
size_t router_scratch_bytes(int T, int H, int E);
// Also clears the status word when p.clear_status is set (the first kernel of a forward).
cudaError_t launch_router(const void* x, const float* Wr, const float* bias, const RouterParams& p,
                          int32_t* topk_ids, float* topk_w, void* scratch, int* status,
                          unsigned long long timeout_ns, cudaStream_t stream);

// ------------------------------------------------------------------ permute
constexpr int PERMUTE_TOK = 256;  // tokens per counting block
constexpr int PERMUTE_SMALL_T = 1024;  // single-CTA permutation up to this many tokens
constexpr int MTILE = 256;        // rows per grouped-GEMM tile (one CTA-pair MMA)

struct PermuteOut {
  int* status;          // DevStatus
  int* blk_hist;        // [nblk, E] scratch
  int* expert_offsets;  // [E+1]
  int* mtile_start;     // [E+1] prefix of ceil(count/MTILE), may be null
  int* row_of;          // [T*k]
  int* tok_of;          // [T*k]
  int* pos_of = nullptr;  // [T*k] or null: slot position t*slot_stride + j of each row
  int slot_stride = 0;    // slots per token in the token-major output buffer
  int extra_rows = 0;     // > 0: one more group of this many rows after the experts
                          // (expert_offsets / mtile_start then have E+2 entries)
  float* w_of;          // [T*k] or null
  void* xp;             // [T*k, H] bf16 or null
  const uint8_t* mask = nullptr;  // [T] or null: tokens with 0 (padding) take no rows
};

cudaError_t launch_permute(const int32_t* topk_ids, const float* topk_w, const void* x, int T,
                           int H, int E, int top_k, const PermuteOut& o, cudaStream_t stream);

// ------------------------------------------------------------------ grouped GEMM
enum EpiKind { EPI_SWIGLU = 0, EPI_ROWSCALE = 1 };

struct GemmArgs {
  // schedule: groups (experts) of rows, each cut into MTILE-row tiles (one per CTA pair)
  const int* mtile_start;  // [num_groups+1] device prefix of tiles per group; null: one group
  const int* row_start;    // [num_groups+1] device first row of each group
  int num_groups;
  int single_rows;         // rows of the only group when mtile_start == null
  int alt_group;           // group read through the second pair of maps (-1: none)
  int alt_rebase;          // 1: its A rows are read at (row - the group's first row),
                           //    e.g. x for the shared expert; 0: at their own row
  int n_tiles;             // output tiles along N
  int k_steps;             // K / 64
  int n_out_tile;          // output columns per tile: 128 (SwiGLU) or 256
  int b_second;            // row offset of the second 128-row half of the B tile
  // epilogue
  __nv_bfloat16* out;      // [rows, ldo]
  int ldo;
  int n_valid;             // valid output columns (N tail mask)
  const float* row_scale;  // EPI_ROWSCALE: weight of each row, or null for 1
  const int* dest_pos;     // EPI_ROWSCALE: output row of each row, or null for
  int dest_mul, dest_add;  //   row * dest_mul + dest_add
  int* status;
  unsigned long long timeout_ns;
};

// A: 2D map over [rows, K] bf16, box 64 x 128, 128B swizzle.
// B: 3D map over [groups, N_rows, K] bf16, box 64 x 128 x 1, 128B swizzle.
cudaError_t make_tmap_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K);
// The same with a box of box_rows rows (the token operand of the swapped GEMM: 32).
cudaError_t make_tmap_2d_box(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K,
                             uint32_t box_rows);
cudaError_t make_tmap_3d(CUtensorMap* map, const void* base, uint64_t groups, uint64_t n_rows,
                         uint64_t K);
// The same with a box of box_rows rows.
cudaError_t make_tmap_3d_box(CUtensorMap* map, const void* base, uint64_t groups,
                             uint64_t n_rows, uint64_t K, uint32_t box_rows);

// tmA2/tmB2 serve group args.alt_group (A rows re-based to 0, B group 0).
cudaError_t launch_grouped_gemm(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB,
                                const CUtensorMap& tmA2, const CUtensorMap& tmB2,
                                const GemmArgs& args, int grid, cudaStream_t stream);

// Swapped operands for few rows per group (grouped_gemm_swap.cu): tmW is the
// weights' 3D map (box 64 x 128 x 1), tmX the rows' 2D map with 32-row boxes;
// groups come from args.row_start (null: one group of args.single_rows rows)
// in chunks of `chunk` (32 or 128) rows; args.n_out_tile must be 128,
// args.n_tiles counts 128-row weight tiles, args.b_second is the up half's
// first row (SwiGLU).
cudaError_t launch_grouped_gemm_swap(int epi, int chunk, const CUtensorMap& tmW,
                                     const CUtensorMap& tmX, const CUtensorMap& tmW2,
                                     const CUtensorMap& tmX2, const GemmArgs& args, int grid,
                                     cudaStream_t stream);

// Both swapped projections in one persistent launch (grouped_gemm_swap_fused.cu):
// up items (args up: EPI_SWIGLU, out = h) then down items (args dn:
// EPI_ROWSCALE, reading h), claimed in order from sched[0]; sched[1 + chunk]
// counts the chunk's finished up-item epilogue warps.  sched (1 + chunks ints)
// must be zero at launch.  maps: w13, xp rows, ws13, x (the shared group's
// rows), w2, h rows, ws2 -- row maps with 32-row boxes, weight maps with
// 128-row boxes.  The shared expert, when present, is group up.alt_group of
// both (its up rows read from x, its down rows from h where they are).
cudaError_t launch_swap_fused(int chunk, const CUtensorMap* maps, const GemmArgs& up,
                              const GemmArgs& dn, int* sched, int grid, cudaStream_t stream);

// FP8 expert weights (grouped_gemm_swap_fp8.cu): UE8M0 scale exponents, one
// per 128 x 128 block, [groups][rows][cols] for the routed experts (s) and
// [rows][cols] for the group args.alt_group (s2); cols = K / 128.
struct Fp8Scales {
  const uint8_t* s;
  const uint8_t* s2;
  int rows;  // scale-block rows per group of s
  int cols;  // scale-block columns (K / 128)
};

// 3D map over [groups, N_rows, K] E4M3 codes (bytes), box 128 x 128 x 1, 128B swizzle.
cudaError_t make_tmap_3d_fp8(CUtensorMap* map, const void* base, uint64_t groups, uint64_t n_rows,
                             uint64_t K);

// The swapped grouped GEMM with FP8 weights: as launch_grouped_gemm_swap, with
// tmW / tmW2 E4M3 maps (make_tmap_3d_fp8) and their block scales in sc; K and
// the weight-row offsets (args.b_second) must be multiples of 128.
cudaError_t launch_grouped_gemm_swap_fp8(int epi, int chunk, const CUtensorMap& tmW,
                                         const CUtensorMap& tmX, const CUtensorMap& tmW2,
                                         const CUtensorMap& tmX2, const GemmArgs& args,
                                         const Fp8Scales& sc, int grid, cudaStream_t stream);

int num_sms();

// ------------------------------------------------------------------ expert parallelism
// ids[r] = the expert whose rows [offsets[e], offsets[e+1]) hold row r + offsets[0].
cudaError_t launch_rows_expert_ids(const int* offsets, int E, int R, int* ids,
                                   cudaStream_t stream);
// tiles[g] = sum over g' < g of ceil((offsets[g'+1] - offsets[g']) / MTILE), g <= groups.
cudaError_t launch_tile_prefix(const int* offsets, int groups, int* tiles, cudaStream_t stream);
// out[t] = bf16( sum_{j<top_k} y[row_of[t*top_k+j]] (0 outside [0, R)) [+ shared[t]]
// [+ residual[t]] ), fp32 in that order.
cudaError_t launch_combine_rows(const void* y, int R, const int* row_of, int top_k, int T, int H,
                                const void* shared, const void* residual, void* out,
                                cudaStream_t stream);

// ------------------------------------------------------------------ misc
cudaError_t launch_rmsnorm(const void* x, const float* gamma, float eps, int T, int H, void* xn,
                           cudaStream_t stream);
// out[t] = bf16( sum_{j<slots} Y[t*slots + j] [+ residual[t]] ), fp32 sum in slot order;
// routed slot j < top_k is skipped when row_of[t*top_k + j] < 0 (a rejected expert id).
cudaError_t launch_combine_slots(const void* Y, const int* row_of, int top_k, int T, int H,
                                 int slots, const void* residual, void* out, cudaStream_t stream);
cudaError_t launch_status_reset(int* status, cudaStream_t stream);
cudaError_t launch_selftest_wait(int* status, unsigned long long timeout_ns, cudaStream_t stream);

}  // namespace rmoe
