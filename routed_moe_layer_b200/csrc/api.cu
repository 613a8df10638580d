// C ABI of libroutedmoe.so (declared in include/routed_moe.h): argument
// checks, workspace layout, tensor-map set-up and the launch sequence of the
// block forward (sglang PR #32341 report, LingBotVideoSparseMoeBlock.forward:
// router -> grouped SwiGLU experts weighted on the output -> fp32 restore ->
// + unscaled shared expert).
#include <stdint.h>
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "routed_moe.h"

using namespace rmoe;

namespace {

constexpr size_t WS_ALIGN = 256;
constexpr unsigned long long DEFAULT_TIMEOUT_NS = 2000000000ull;  // 2 s
constexpr int MAX_E = 128;
constexpr int MAX_TOPK = 16;
constexpr int MAX_NGROUP = 16;  // the router ranks groups within a half warp
constexpr int MAX_DIM = 16384;

size_t align_up(size_t v) { return (v + WS_ALIGN - 1) & ~(WS_ALIGN - 1); }

int32_t check_cfg(const moe_cfg_t* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->H <= 0 || c->E <= 0 || c->I <= 0 || c->I_shared < 0 || c->top_k <= 0 ||
      c->n_group <= 0 || c->topk_group <= 0 || c->flags != 0)
    return MOE_ERR_INVALID_ARG;
  if (!(c->routed_scaling_factor == c->routed_scaling_factor)) return MOE_ERR_INVALID_ARG;
  if (c->norm_topk_prob != 0 && c->norm_topk_prob != 1) return MOE_ERR_INVALID_ARG;
  // the group-limited top-k assumes E divisible by n_group and, when groups
  // are actually dropped, at least two experts per group (the per-group top-2)
  if (c->E % c->n_group != 0) return MOE_ERR_INVALID_ARG;
  if (c->topk_group > c->n_group) return MOE_ERR_INVALID_ARG;
  const int gs = c->E / c->n_group;
  if (c->topk_group < c->n_group && gs < 2) return MOE_ERR_INVALID_ARG;
  if ((int64_t)c->topk_group * gs < c->top_k) return MOE_ERR_INVALID_ARG;
  if (c->E > MAX_E || c->top_k > MAX_TOPK || c->n_group > MAX_NGROUP)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->H % 64 != 0 || c->I % 64 != 0 || c->I_shared % 64 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->H > MAX_DIM || c->I > MAX_DIM || c->I_shared > MAX_DIM) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)c->T * c->top_k > (int64_t)INT32_MAX / 2) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

struct FwdLayout {
  size_t status, router, ids, w, blk_hist, offsets, mtiles, row_of, tok_of, w_of, pos_of, y, h,
      hs, sched, y_sep, total;
};

// Slots per token of the token-major buffer of weighted expert outputs: the
// routed experts, then the shared expert.
int slots_per_token(const moe_cfg_t& c) { return c.top_k + (c.I_shared > 0 ? 1 : 0); }

// With I_shared == I the shared expert runs as one more group (number E) of
// the routed grouped GEMMs: its rows follow the R routed rows in h, its A rows
// come from x and its weights from ws13 / ws2.
bool fuse_shared(const moe_cfg_t& c) { return c.I_shared > 0 && c.I_shared == c.I; }

// Few rows per expert (at most 64 on average): the grouped GEMMs run with
// swapped operands (weight rows on the MMA's M, the expert's rows on N), so
// that tiles are not padded to 256 rows.  Decided from the shapes only.
bool use_swap(const moe_cfg_t& c) { return (int64_t)c.T * c.top_k <= 64LL * c.E; }

// Token rows per item of the swapped GEMMs: 32 when the experts average at
// most 20 rows (so that few of them need a second chunk), else 128.
int swap_chunk(const moe_cfg_t& c) { return (int64_t)c.T * c.top_k <= 20LL * c.E ? 32 : 128; }

// Upper bound on the swapped GEMMs' chunks: every group adds at most one partial chunk.
long long swap_chunk_bound(const moe_cfg_t& c) {
  const long long R = (long long)c.T * c.top_k;
  return R / swap_chunk(c) + c.E + (fuse_shared(c) ? 1 : 0) + 1;
}

// The swapped up and down projections run as one launch (grouped_gemm_swap_fused.cu)
// when the shared expert, if any, is a group of them.
bool fused_swap(const moe_cfg_t& c) { return use_swap(c) && (fuse_shared(c) || c.I_shared == 0); }

FwdLayout fwd_layout(const moe_cfg_t& c) {
  FwdLayout L;
  const size_t T = c.T, R = T * c.top_k, E = c.E;
  const size_t nblk = (T + PERMUTE_TOK - 1) / PERMUTE_TOK;
  size_t off = 0;
  L.status = off;   off += align_up(sizeof(DevStatus));
  L.router = off;   off += align_up(router_scratch_bytes(c.T, c.H, c.E));
  L.ids = off;      off += align_up(R * 4);
  L.w = off;        off += align_up(R * 4);
  L.blk_hist = off; off += align_up(nblk * E * 4);
  L.offsets = off;  off += align_up((E + 2) * 4);
  L.mtiles = off;   off += align_up((E + 2) * 4);
  L.row_of = off;   off += align_up(R * 4);
  L.tok_of = off;   off += align_up(R * 4);
  L.w_of = off;     off += align_up(R * 4);
  L.pos_of = off;   off += align_up(R * 4);
  // gathered expert rows [R, H]; once the up projection has read them, the same
  // bytes hold the weighted expert outputs in token-major slot order [T*slots, H]
  L.y = off;        off += align_up(std::max(R, T * (size_t)slots_per_token(c)) * c.H * 2);
  L.h = off;        off += align_up((R + (fuse_shared(c) ? T : 0)) * c.I * 2);
  L.hs = off;       off += align_up(fuse_shared(c) ? 0 : T * c.I_shared * 2);
  // fused swapped projections: the item claim counter, then one ready counter per chunk;
  // and a buffer of their own for the weighted outputs, which the down items write while
  // other CTAs' up items may still read the gathered rows
  L.sched = off;    off += align_up(fused_swap(c) ? (1 + swap_chunk_bound(c)) * 4 : 0);
  L.y_sep = off;
  off += align_up(fused_swap(c) ? T * (size_t)slots_per_token(c) * c.H * 2 : 0);
  L.total = off;
  return L;
}

struct PermLayout {
  size_t status, blk_hist, mtiles, total;
};

PermLayout perm_layout(const moe_cfg_t& c) {
  PermLayout L;
  const size_t nblk = ((size_t)c.T + PERMUTE_TOK - 1) / PERMUTE_TOK;
  size_t off = 0;
  L.status = off;   off += align_up(sizeof(DevStatus));
  L.blk_hist = off; off += align_up(nblk * c.E * 4);
  L.mtiles = off;   off += align_up((c.E + 1) * 4);
  L.total = off;
  return L;
}

bool ws_ok(const void* ws, size_t have, size_t need) {
  if (need == 0) return true;
  if (!ws || have < need) return false;
  return (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN) == 0;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

int32_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

RouterParams router_params(const moe_cfg_t& c) {
  RouterParams p;
  p.T = c.T;
  p.H = c.H;
  p.E = c.E;
  p.top_k = c.top_k;
  p.n_group = c.n_group;
  p.topk_group = c.topk_group;
  p.norm_topk_prob = c.norm_topk_prob;
  p.rsf = c.routed_scaling_factor;
  p.clear_status = 1;
  return p;
}

#define RMOE_TRY(expr)                       \
  do {                                       \
    const cudaError_t e_ = (expr);           \
    if (e_ != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

// Host checks of moe_forward (the configuration already checked).
int32_t check_forward_args(const moe_cfg_t& c, const void* x, const float* Wr, const float* bias,
                           const void* w13, const void* w2, const void* ws13, const void* ws2,
                           const void* out, const moe_forward_opts_t* opts) {
  if (!x || !Wr || !bias || !w13 || !w2 || !out) return MOE_ERR_INVALID_ARG;
  if ((c.I_shared > 0) != (ws13 != nullptr && ws2 != nullptr)) return MOE_ERR_INVALID_ARG;
  if (out == x) return MOE_ERR_INVALID_ARG;
  if (opts && opts->wait_timeout_ns < 0) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// The expert and shared-expert GEMMs with swapped operands (use_swap).
template <typename Rec>
cudaError_t swap_gemms(const moe_cfg_t& c, const void* x, __nv_bfloat16* xp, __nv_bfloat16* h,
                       __nv_bfloat16* hs, __nv_bfloat16* Y, const CUtensorMap& tm_w13,
                       const CUtensorMap& tm_w2, const CUtensorMap& tm_ws13,
                       const CUtensorMap& tm_ws2, const int* offsets, const PermuteOut& o,
                       const GemmArgs& a, int* sched, int sms, Rec& record, cudaStream_t s) {
  const size_t T = c.T, R = T * c.top_k;
  const int slots = slots_per_token(c);
  const bool fused = fuse_shared(c);
  const int groups = c.E + (fused ? 1 : 0);
  const int chunk = swap_chunk(c);
  const long long chunk_bound = (long long)(R / chunk) + groups + 1;
  // h holds the routed rows, then (fused) the shared group's T rows; the
  // shared group starts at expert_offsets[E], which is below T*top_k when
  // rows are dropped (padding tokens, rejected ids), so the down projection
  // reads the shared rows where they are, through the map of all of h
  const size_t h_rows = R + (fused ? T : 0);
  CUtensorMap tm_xp, tm_x, tm_h, tm_hs;
  cudaError_t e;
  if ((e = make_tmap_2d_box(&tm_xp, xp, R, c.H, 32)) != cudaSuccess) return e;
  if ((e = make_tmap_2d_box(&tm_h, h, h_rows, c.I, 32)) != cudaSuccess) return e;
  tm_x = tm_hs = tm_xp;  // unused unless there is a shared expert
  if (c.I_shared > 0) {
    if ((e = make_tmap_2d_box(&tm_x, x, T, c.H, 32)) != cudaSuccess) return e;
    if (!fused && (e = make_tmap_2d_box(&tm_hs, hs, T, c.I_shared, 32)) != cudaSuccess) return e;
  }
  // h[r, i] = silu(W13g[i] . x_r) * (W13u[i] . x_r) per group (shared expert: group E)
  GemmArgs gu = a;
  gu.mtile_start = o.mtile_start;
  gu.row_start = offsets;
  gu.num_groups = groups;
  if (fused) {  // shared rows: A from x at (row - group start)
    gu.alt_group = c.E;
    gu.alt_rebase = 1;
  }
  gu.n_tiles = (c.I + 127) / 128;
  gu.k_steps = c.H / 64;
  gu.n_out_tile = 128;
  gu.b_second = c.I;
  gu.out = h;
  gu.ldo = c.I;
  gu.n_valid = c.I;
  // Y[pos_r, n] = w_r * (W2[n] . h_r) per expert; shared rows to slot top_k, unscaled
  GemmArgs gd = a;
  gd.mtile_start = o.mtile_start;
  gd.row_start = offsets;
  gd.num_groups = groups;
  if (fused) {  // shared rows: A from h at their own rows, weights ws2, unscaled
    gd.alt_group = c.E;
    gd.alt_rebase = 0;
  }
  gd.n_tiles = (c.H + 127) / 128;
  gd.k_steps = c.I / 64;
  gd.n_out_tile = 128;
  gd.out = Y;
  gd.ldo = c.H;
  gd.n_valid = c.H;
  gd.row_scale = o.w_of;
  gd.dest_pos = o.pos_of;
  gd.dest_mul = slots;
  gd.dest_add = c.top_k;
  if ((e = record(MOE_STAGE_EXPERT_UP)) != cudaSuccess) return e;
  if (sched) {  // both projections in one launch (the expert_down stage is then empty)
    const CUtensorMap maps[7] = {tm_w13, tm_xp, tm_ws13, tm_x, tm_w2, tm_h, tm_ws2};
    const int grid =
        (int)std::min<long long>(sms, chunk_bound * (gu.n_tiles + (long long)gd.n_tiles));
    if ((e = launch_swap_fused(chunk, maps, gu, gd, sched, grid, s)) != cudaSuccess) return e;
    if ((e = record(MOE_STAGE_EXPERT_DOWN)) != cudaSuccess) return e;
  } else {
    const int grid_u = (int)std::min<long long>(sms, chunk_bound * gu.n_tiles);
    if ((e = launch_grouped_gemm_swap(EPI_SWIGLU, chunk, tm_w13, tm_xp, tm_ws13, tm_x, gu,
                                      grid_u, s)) != cudaSuccess)
      return e;
    if ((e = record(MOE_STAGE_EXPERT_DOWN)) != cudaSuccess) return e;
    const int grid_d = (int)std::min<long long>(sms, chunk_bound * gd.n_tiles);
    if ((e = launch_grouped_gemm_swap(EPI_ROWSCALE, chunk, tm_w2, tm_h, tm_ws2, tm_h, gd, grid_d,
                                      s)) != cudaSuccess)
      return e;
  }
  if ((e = record(MOE_STAGE_SHARED_EXPERT)) != cudaSuccess) return e;
  if (c.I_shared > 0 && !fused) {
    const long long chunks = (long long)(T + chunk - 1) / chunk;
    {  // hs = silu(x . Ws13g^T) * (x . Ws13u^T)
      GemmArgs g = a;
      g.single_rows = c.T;
      g.n_tiles = (c.I_shared + 127) / 128;
      g.k_steps = c.H / 64;
      g.n_out_tile = 128;
      g.b_second = c.I_shared;
      g.out = hs;
      g.ldo = c.I_shared;
      g.n_valid = c.I_shared;
      const int grid = (int)std::min<long long>(sms, chunks * g.n_tiles);
      if ((e = launch_grouped_gemm_swap(EPI_SWIGLU, chunk, tm_ws13, tm_x, tm_ws13, tm_x, g, grid,
                                        s)) !=
          cudaSuccess)
        return e;
    }
    {  // Y[t*slots + top_k] = hs . Ws2^T  (unscaled)
      GemmArgs g = a;
      g.single_rows = c.T;
      g.n_tiles = (c.H + 127) / 128;
      g.k_steps = c.I_shared / 64;
      g.n_out_tile = 128;
      g.out = Y;
      g.ldo = c.H;
      g.n_valid = c.H;
      g.dest_mul = slots;
      g.dest_add = c.top_k;
      const int grid = (int)std::min<long long>(sms, chunks * g.n_tiles);
      if ((e = launch_grouped_gemm_swap(EPI_ROWSCALE, chunk, tm_ws2, tm_hs, tm_ws2, tm_hs, g,
                                        grid, s)) !=
          cudaSuccess)
        return e;
    }
  }
  return cudaSuccess;
}

// The launch sequence of one block forward; arguments already checked, T > 0.
// clear_status: the router's first kernel clears the status word.
int32_t forward_impl(const void* x, const float* Wr, const float* bias, const void* w13,
                     const void* w2, const void* ws13, const void* ws2, const moe_cfg_t& c,
                     void* out, const moe_forward_opts_t* opts, void* workspace, bool clear_status,
                     cudaStream_t s) {
  const FwdLayout L = fwd_layout(c);
  void** ev = opts ? opts->stage_events : nullptr;
  const unsigned long long timeout =
      (opts && opts->wait_timeout_ns > 0) ? (unsigned long long)opts->wait_timeout_ns
                                          : DEFAULT_TIMEOUT_NS;
  const size_t T = c.T, R = T * c.top_k;
  int* status = at<int>(workspace, L.status);
  int32_t* ids = (opts && opts->topk_ids) ? opts->topk_ids : at<int32_t>(workspace, L.ids);
  float* tw = (opts && opts->topk_w) ? opts->topk_w : at<float>(workspace, L.w);
  int* offsets = at<int>(workspace, L.offsets);
  int* mtiles = at<int>(workspace, L.mtiles);
  int* row_of = at<int>(workspace, L.row_of);
  __nv_bfloat16* xp = at<__nv_bfloat16>(workspace, L.y);  // gathered rows, then ...
  // ... token-major weighted outputs (once the up projection has read them; in the
  // fused swapped launch both run at once, so the outputs get a buffer of their own)
  __nv_bfloat16* Y = fused_swap(c) ? at<__nv_bfloat16>(workspace, L.y_sep) : xp;
  __nv_bfloat16* h = at<__nv_bfloat16>(workspace, L.h);
  __nv_bfloat16* hs = at<__nv_bfloat16>(workspace, L.hs);

  // tensor maps (host-side descriptors, passed by value to the kernels)
  const int slots = slots_per_token(c);
  const bool fused = fuse_shared(c);
  const size_t h_rows = R + (fused ? T : 0);
  CUtensorMap tm_xp, tm_w13, tm_h, tm_w2, tm_x, tm_ws13, tm_hs, tm_ws2;
  RMOE_TRY(make_tmap_2d(&tm_xp, xp, R, c.H));
  RMOE_TRY(make_tmap_3d(&tm_w13, w13, c.E, 2 * (uint64_t)c.I, c.H));
  // all of h: the routed rows, then (fused) the shared group's T rows, which
  // start at expert_offsets[E] -- below T*top_k when rows are dropped (padding
  // tokens, rejected ids) -- and are read where they are
  RMOE_TRY(make_tmap_2d(&tm_h, h, h_rows, c.I));
  RMOE_TRY(make_tmap_3d(&tm_w2, w2, c.E, c.H, c.I));
  if (c.I_shared > 0) {
    RMOE_TRY(make_tmap_2d(&tm_x, x, T, c.H));
    RMOE_TRY(make_tmap_3d(&tm_ws13, ws13, 1, 2 * (uint64_t)c.I_shared, c.H));
    RMOE_TRY(make_tmap_3d(&tm_ws2, ws2, 1, c.H, c.I_shared));
    if (!fused) RMOE_TRY(make_tmap_2d(&tm_hs, hs, T, c.I_shared));
  } else {
    tm_x = tm_ws13 = tm_ws2 = tm_xp;  // unused second maps
  }
  const int sms = num_sms();

  auto record = [&](int i) -> cudaError_t {
    return (ev && ev[i]) ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) : cudaSuccess;
  };

  RMOE_TRY(record(MOE_STAGE_ROUTER));
  RouterParams rp = router_params(c);
  rp.clear_status = clear_status ? 1 : 0;
  rp.mask = opts ? opts->token_mask : nullptr;
  int* sched = fused_swap(c) ? at<int>(workspace, L.sched) : nullptr;
  if (sched) {  // the fused swapped projections' counters start at zero
    rp.zero = sched;
    rp.zero_n = (int)(1 + swap_chunk_bound(c));
  }
  RMOE_TRY(launch_router(x, Wr, bias, rp, ids, tw, at<void>(workspace, L.router), status, timeout,
                         s));

  RMOE_TRY(record(MOE_STAGE_PERMUTE));
  PermuteOut o;
  o.status = status;
  o.blk_hist = at<int>(workspace, L.blk_hist);
  o.expert_offsets = offsets;
  o.mtile_start = mtiles;
  o.row_of = row_of;
  o.tok_of = at<int>(workspace, L.tok_of);
  o.w_of = at<float>(workspace, L.w_of);
  o.pos_of = at<int>(workspace, L.pos_of);
  o.slot_stride = slots;
  o.extra_rows = fused ? c.T : 0;
  o.xp = xp;
  o.mask = rp.mask;
  RMOE_TRY(launch_permute(ids, tw, x, c.T, c.H, c.E, c.top_k, o, s));
  const void* residual = opts ? opts->residual : nullptr;

  // tiles of MTILE rows, each computed by a pair of CTAs; every group adds at
  // most one partial tile
  const int groups = c.E + (fused ? 1 : 0);
  const long long mt_bound = (long long)(h_rows / MTILE) + groups;
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.status = status;
  a.timeout_ns = timeout;
  a.alt_group = -1;

  if (use_swap(c)) {
    RMOE_TRY(swap_gemms(c, x, xp, h, hs, Y, tm_w13, tm_w2, tm_ws13, tm_ws2, offsets, o, a, sched,
                        sms, record, s));
  } else {
    RMOE_TRY(record(MOE_STAGE_EXPERT_UP));
    {  // h = silu(A . W13g^T) * (A . W13u^T) per group: A = gathered rows (experts), x (shared)
      GemmArgs g = a;
      g.mtile_start = mtiles;
      g.row_start = offsets;
      g.num_groups = groups;
      if (fused) {  // shared rows: A from x at (row - group start)
        g.alt_group = c.E;
        g.alt_rebase = 1;
      }
      g.n_tiles = (c.I + 127) / 128;
      g.k_steps = c.H / 64;
      g.n_out_tile = 128;
      g.b_second = c.I;
      g.out = h;
      g.ldo = c.I;
      g.n_valid = c.I;
      const int grid = (int)std::min<long long>(sms, 2LL * mt_bound * g.n_tiles);
      RMOE_TRY(launch_grouped_gemm(EPI_SWIGLU, tm_xp, tm_w13, tm_x, tm_ws13, g, grid, s));
    }
    RMOE_TRY(record(MOE_STAGE_EXPERT_DOWN));
    {  // Y[t*slots + j] = w_tj * (h . W2^T) per expert; shared rows to slot top_k, unscaled
      GemmArgs g = a;
      g.mtile_start = mtiles;
      g.row_start = offsets;
      g.num_groups = groups;
      if (fused) {  // shared rows: A from h at their own rows, weights ws2, unscaled
        g.alt_group = c.E;
        g.alt_rebase = 0;
      }
      g.n_tiles = (c.H + 255) / 256;
      g.k_steps = c.I / 64;
      g.n_out_tile = 256;
      g.b_second = 128;
      g.out = Y;
      g.ldo = c.H;
      g.n_valid = c.H;
      g.row_scale = o.w_of;
      g.dest_pos = o.pos_of;
      g.dest_mul = slots;
      g.dest_add = c.top_k;
      const int grid = (int)std::min<long long>(sms, 2LL * mt_bound * g.n_tiles);
      RMOE_TRY(launch_grouped_gemm(EPI_ROWSCALE, tm_h, tm_w2, tm_h, tm_ws2, g, grid, s));
    }
    RMOE_TRY(record(MOE_STAGE_SHARED_EXPERT));
    if (c.I_shared > 0 && !fused) {
      {  // hs = silu(x . Ws13g^T) * (x . Ws13u^T)
        GemmArgs g = a;
        g.single_rows = c.T;
        g.n_tiles = (c.I_shared + 127) / 128;
        g.k_steps = c.H / 64;
        g.n_out_tile = 128;
        g.b_second = c.I_shared;
        g.out = hs;
        g.ldo = c.I_shared;
        g.n_valid = c.I_shared;
        const int tiles = (int)((T + MTILE - 1) / MTILE) * g.n_tiles;
        RMOE_TRY(launch_grouped_gemm(EPI_SWIGLU, tm_x, tm_ws13, tm_x, tm_ws13, g,
                                     std::min(sms, 2 * tiles), s));
      }
      {  // Y[t*slots + top_k] = hs . Ws2^T  (unscaled)
        GemmArgs g = a;
        g.single_rows = c.T;
        g.n_tiles = (c.H + 255) / 256;
        g.k_steps = c.I_shared / 64;
        g.n_out_tile = 256;
        g.b_second = 128;
        g.out = Y;
        g.ldo = c.H;
        g.n_valid = c.H;
        g.dest_mul = slots;
        g.dest_add = c.top_k;
        const int tiles = (int)((T + MTILE - 1) / MTILE) * g.n_tiles;
        RMOE_TRY(launch_grouped_gemm(EPI_ROWSCALE, tm_hs, tm_ws2, tm_hs, tm_ws2, g,
                                     std::min(sms, 2 * tiles), s));
      }
    }
  }
  RMOE_TRY(record(MOE_STAGE_COMBINE));
  RMOE_TRY(launch_combine_slots(Y, row_of, c.top_k, c.T, c.H, slots, residual, out, s));
  RMOE_TRY(record(MOE_NUM_STAGES));
  return MOE_OK;
}

// The expert and shared-expert GEMMs with FP8 weights: the swapped kernels
// with weight tiles dequantised in shared memory (grouped_gemm_swap_fp8.cu).
struct Fp8Weights {
  const uint8_t *w13_q, *w13_s, *w2_q, *w2_s, *ws13_q, *ws13_s, *ws2_q, *ws2_s;
};

template <typename Rec>
cudaError_t swap_gemms_fp8(const moe_cfg_t& c, const void* x, __nv_bfloat16* xp,
                           __nv_bfloat16* h, __nv_bfloat16* hs, __nv_bfloat16* Y,
                           const Fp8Weights& fw, const int* offsets, const PermuteOut& o,
                           const GemmArgs& a, int sms, Rec& record, cudaStream_t s) {
  const size_t T = c.T, R = T * c.top_k;
  const int slots = slots_per_token(c);
  const bool fused = fuse_shared(c);
  const int groups = c.E + (fused ? 1 : 0);
  const int chunk = swap_chunk(c);
  const long long chunk_bound = (long long)(R / chunk) + groups + 1;
  const size_t h_rows = R + (fused ? T : 0);
  CUtensorMap tm_xp, tm_x, tm_h, tm_hs, tm_w13, tm_w2, tm_ws13, tm_ws2;
  cudaError_t e;
  if ((e = make_tmap_2d_box(&tm_xp, xp, R, c.H, 32)) != cudaSuccess) return e;
  if ((e = make_tmap_2d_box(&tm_h, h, h_rows, c.I, 32)) != cudaSuccess) return e;
  if ((e = make_tmap_3d_fp8(&tm_w13, fw.w13_q, c.E, 2 * (uint64_t)c.I, c.H)) != cudaSuccess)
    return e;
  if ((e = make_tmap_3d_fp8(&tm_w2, fw.w2_q, c.E, c.H, c.I)) != cudaSuccess) return e;
  tm_x = tm_hs = tm_xp;  // unused unless there is a shared expert
  tm_ws13 = tm_w13;
  tm_ws2 = tm_w2;
  if (c.I_shared > 0) {
    if ((e = make_tmap_2d_box(&tm_x, x, T, c.H, 32)) != cudaSuccess) return e;
    if (!fused && (e = make_tmap_2d_box(&tm_hs, hs, T, c.I_shared, 32)) != cudaSuccess) return e;
    if ((e = make_tmap_3d_fp8(&tm_ws13, fw.ws13_q, 1, 2 * (uint64_t)c.I_shared, c.H)) !=
        cudaSuccess)
      return e;
    if ((e = make_tmap_3d_fp8(&tm_ws2, fw.ws2_q, 1, c.H, c.I_shared)) != cudaSuccess) return e;
  }
  const Fp8Scales up_sc{fw.w13_s, fw.ws13_s, 2 * c.I / 128, c.H / 128};
  const Fp8Scales down_sc{fw.w2_s, fw.ws2_s, c.H / 128, c.I / 128};
  if ((e = record(MOE_STAGE_EXPERT_UP)) != cudaSuccess) return e;
  {  // h[r, i] = silu(W13g[i] . x_r) * (W13u[i] . x_r) per group (shared expert: group E)
    GemmArgs g = a;
    g.mtile_start = o.mtile_start;
    g.row_start = offsets;
    g.num_groups = groups;
    if (fused) {
      g.alt_group = c.E;
      g.alt_rebase = 1;
    }
    g.n_tiles = c.I / 128;
    g.k_steps = c.H / 64;
    g.n_out_tile = 128;
    g.b_second = c.I;
    g.out = h;
    g.ldo = c.I;
    g.n_valid = c.I;
    const int grid = (int)std::min<long long>(sms, chunk_bound * g.n_tiles);
    if ((e = launch_grouped_gemm_swap_fp8(EPI_SWIGLU, chunk, tm_w13, tm_xp, tm_ws13, tm_x, g,
                                          up_sc, grid, s)) != cudaSuccess)
      return e;
  }
  if ((e = record(MOE_STAGE_EXPERT_DOWN)) != cudaSuccess) return e;
  {  // Y[pos_r, n] = w_r * (W2[n] . h_r) per expert; shared rows to slot top_k, unscaled
    GemmArgs g = a;
    g.mtile_start = o.mtile_start;
    g.row_start = offsets;
    g.num_groups = groups;
    if (fused) {
      g.alt_group = c.E;
      g.alt_rebase = 0;
    }
    g.n_tiles = c.H / 128;
    g.k_steps = c.I / 64;
    g.n_out_tile = 128;
    g.out = Y;
    g.ldo = c.H;
    g.n_valid = c.H;
    g.row_scale = o.w_of;
    g.dest_pos = o.pos_of;
    g.dest_mul = slots;
    g.dest_add = c.top_k;
    const int grid = (int)std::min<long long>(sms, chunk_bound * g.n_tiles);
    if ((e = launch_grouped_gemm_swap_fp8(EPI_ROWSCALE, chunk, tm_w2, tm_h, tm_ws2, tm_h, g,
                                          down_sc, grid, s)) != cudaSuccess)
      return e;
  }
  if ((e = record(MOE_STAGE_SHARED_EXPERT)) != cudaSuccess) return e;
  if (c.I_shared > 0 && !fused) {
    const long long chunks = (long long)(T + chunk - 1) / chunk;
    {  // hs = silu(x . Ws13g^T) * (x . Ws13u^T)
      GemmArgs g = a;
      g.single_rows = c.T;
      g.n_tiles = c.I_shared / 128;
      g.k_steps = c.H / 64;
      g.n_out_tile = 128;
      g.b_second = c.I_shared;
      g.out = hs;
      g.ldo = c.I_shared;
      g.n_valid = c.I_shared;
      const Fp8Scales sc{fw.ws13_s, nullptr, 2 * c.I_shared / 128, c.H / 128};
      const int grid = (int)std::min<long long>(sms, chunks * g.n_tiles);
      if ((e = launch_grouped_gemm_swap_fp8(EPI_SWIGLU, chunk, tm_ws13, tm_x, tm_ws13, tm_x, g,
                                            sc, grid, s)) != cudaSuccess)
        return e;
    }
    {  // Y[t*slots + top_k] = hs . Ws2^T  (unscaled)
      GemmArgs g = a;
      g.single_rows = c.T;
      g.n_tiles = c.H / 128;
      g.k_steps = c.I_shared / 64;
      g.n_out_tile = 128;
      g.out = Y;
      g.ldo = c.H;
      g.n_valid = c.H;
      g.dest_mul = slots;
      g.dest_add = c.top_k;
      const Fp8Scales sc{fw.ws2_s, nullptr, c.H / 128, c.I_shared / 128};
      const int grid = (int)std::min<long long>(sms, chunks * g.n_tiles);
      if ((e = launch_grouped_gemm_swap_fp8(EPI_ROWSCALE, chunk, tm_ws2, tm_hs, tm_ws2, tm_hs, g,
                                            sc, grid, s)) != cudaSuccess)
        return e;
    }
  }
  return cudaSuccess;
}

// The launch sequence of the block forward with FP8 expert weights: the
// router, permutation and combine of forward_impl around swap_gemms_fp8.
int32_t forward_fp8_impl(const void* x, const float* Wr, const float* bias, const Fp8Weights& fw,
                         const moe_cfg_t& c, void* out, const moe_forward_opts_t* opts,
                         void* workspace, cudaStream_t s) {
  const FwdLayout L = fwd_layout(c);
  void** ev = opts ? opts->stage_events : nullptr;
  const unsigned long long timeout =
      (opts && opts->wait_timeout_ns > 0) ? (unsigned long long)opts->wait_timeout_ns
                                          : DEFAULT_TIMEOUT_NS;
  int* status = at<int>(workspace, L.status);
  int32_t* ids = (opts && opts->topk_ids) ? opts->topk_ids : at<int32_t>(workspace, L.ids);
  float* tw = (opts && opts->topk_w) ? opts->topk_w : at<float>(workspace, L.w);
  int* offsets = at<int>(workspace, L.offsets);
  int* row_of = at<int>(workspace, L.row_of);
  __nv_bfloat16* xp = at<__nv_bfloat16>(workspace, L.y);
  __nv_bfloat16* Y = xp;
  __nv_bfloat16* h = at<__nv_bfloat16>(workspace, L.h);
  __nv_bfloat16* hs = at<__nv_bfloat16>(workspace, L.hs);
  const int slots = slots_per_token(c);
  const bool fused = fuse_shared(c);
  const int sms = num_sms();
  auto record = [&](int i) -> cudaError_t {
    return (ev && ev[i]) ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) : cudaSuccess;
  };

  RMOE_TRY(record(MOE_STAGE_ROUTER));
  RouterParams rp = router_params(c);
  rp.mask = opts ? opts->token_mask : nullptr;
  RMOE_TRY(launch_router(x, Wr, bias, rp, ids, tw, at<void>(workspace, L.router), status, timeout,
                         s));
  RMOE_TRY(record(MOE_STAGE_PERMUTE));
  PermuteOut o;
  o.status = status;
  o.blk_hist = at<int>(workspace, L.blk_hist);
  o.expert_offsets = offsets;
  o.mtile_start = at<int>(workspace, L.mtiles);
  o.row_of = row_of;
  o.tok_of = at<int>(workspace, L.tok_of);
  o.w_of = at<float>(workspace, L.w_of);
  o.pos_of = at<int>(workspace, L.pos_of);
  o.slot_stride = slots;
  o.extra_rows = fused ? c.T : 0;
  o.xp = xp;
  o.mask = rp.mask;
  RMOE_TRY(launch_permute(ids, tw, x, c.T, c.H, c.E, c.top_k, o, s));
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.status = status;
  a.timeout_ns = timeout;
  a.alt_group = -1;
  RMOE_TRY(swap_gemms_fp8(c, x, xp, h, hs, Y, fw, offsets, o, a, sms, record, s));
  RMOE_TRY(record(MOE_STAGE_COMBINE));
  const void* residual = opts ? opts->residual : nullptr;
  RMOE_TRY(launch_combine_slots(Y, row_of, c.top_k, c.T, c.H, slots, residual, out, s));
  RMOE_TRY(record(MOE_NUM_STAGES));
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(int32_t status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument or configuration";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE: shape outside the kernels' limits";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT: a device-side wait ran out";
    case MOE_ERR_DEVICE_INDEX: return "MOE_ERR_DEVICE_INDEX: an expert id outside [0, E)";
    case MOE_ERR_NO_DEVICE: return "MOE_ERR_NO_DEVICE: no usable CUDA device";
    default: return "unknown moe_status_t";
  }
}

int32_t moe_check_config(const moe_cfg_t* cfg) { return check_cfg(cfg); }

size_t moe_route_workspace_bytes(const moe_cfg_t* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return align_up(sizeof(DevStatus)) + align_up(router_scratch_bytes(cfg->T, cfg->H, cfg->E));
}

size_t moe_permute_workspace_bytes(const moe_cfg_t* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return perm_layout(*cfg).total;
}

size_t moe_workspace_bytes(const moe_cfg_t* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return fwd_layout(*cfg).total;
}

int32_t moe_route_masked(const void* x, const float* Wr, const float* bias,
                         const uint8_t* token_mask, const moe_cfg_t* cfg, int32_t* topk_ids,
                         float* topk_w, void* workspace, size_t workspace_bytes, void* stream) {
  const int32_t st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !Wr || !bias || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!ws_ok(workspace, workspace_bytes, moe_route_workspace_bytes(cfg))) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = at<int>(workspace, 0);
  RouterParams rp = router_params(*cfg);
  rp.mask = token_mask;
  return cuda_status(launch_router(x, Wr, bias, rp, topk_ids, topk_w,
                                   at<void>(workspace, align_up(sizeof(DevStatus))), status,
                                   DEFAULT_TIMEOUT_NS, s));
}

int32_t moe_route(const void* x, const float* Wr, const float* bias, const moe_cfg_t* cfg,
                  int32_t* topk_ids, float* topk_w, void* workspace, size_t workspace_bytes,
                  void* stream) {
  return moe_route_masked(x, Wr, bias, nullptr, cfg, topk_ids, topk_w, workspace,
                          workspace_bytes, stream);
}

int32_t moe_permute(const int32_t* topk_ids, const float* topk_w, const void* x,
                    const moe_cfg_t* cfg, int32_t* expert_offsets, int32_t* row_of,
                    int32_t* tok_of, float* w_of, void* xp, void* workspace,
                    size_t workspace_bytes, void* stream) {
  const int32_t st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!topk_ids || !expert_offsets || !row_of || !tok_of) return MOE_ERR_INVALID_ARG;
  if (xp && !x) return MOE_ERR_INVALID_ARG;
  const PermLayout L = perm_layout(*cfg);
  if (!ws_ok(workspace, workspace_bytes, L.total)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = at<int>(workspace, L.status);
  RMOE_TRY(launch_status_reset(status, s));
  PermuteOut o;
  o.status = status;
  o.blk_hist = at<int>(workspace, L.blk_hist);
  o.expert_offsets = expert_offsets;
  o.mtile_start = at<int>(workspace, L.mtiles);
  o.row_of = row_of;
  o.tok_of = tok_of;
  o.w_of = w_of;
  o.xp = xp;
  return cuda_status(launch_permute(topk_ids, topk_w, x, cfg->T, cfg->H, cfg->E, cfg->top_k, o, s));
}

int32_t moe_forward(const void* x, const float* Wr, const float* bias, const void* w13,
                    const void* w2, const void* ws13, const void* ws2, const moe_cfg_t* cfg,
                    void* out, const moe_forward_opts_t* opts, void* workspace,
                    size_t workspace_bytes, void* stream) {
  const int32_t st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  const moe_cfg_t& c = *cfg;
  if (c.T == 0) return MOE_OK;
  const int32_t a = check_forward_args(c, x, Wr, bias, w13, w2, ws13, ws2, out, opts);
  if (a != MOE_OK) return a;
  if (!ws_ok(workspace, workspace_bytes, fwd_layout(c).total)) return MOE_ERR_WORKSPACE;
  return forward_impl(x, Wr, bias, w13, w2, ws13, ws2, c, out, opts, workspace, true,
                      static_cast<cudaStream_t>(stream));
}

int32_t moe_forward_fp8(const void* x, const float* Wr, const float* bias, const uint8_t* w13_q,
                        const uint8_t* w13_s, const uint8_t* w2_q, const uint8_t* w2_s,
                        const uint8_t* ws13_q, const uint8_t* ws13_s, const uint8_t* ws2_q,
                        const uint8_t* ws2_s, const moe_cfg_t* cfg, void* out,
                        const moe_forward_opts_t* opts, void* workspace, size_t workspace_bytes,
                        void* stream) {
  const int32_t st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  const moe_cfg_t& c = *cfg;
  if (c.H % 128 != 0 || c.I % 128 != 0 || c.I_shared % 128 != 0)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (c.T == 0) return MOE_OK;
  if (!w13_s || !w2_s) return MOE_ERR_INVALID_ARG;
  if ((c.I_shared > 0) != (ws13_s != nullptr && ws2_s != nullptr)) return MOE_ERR_INVALID_ARG;
  const int32_t a = check_forward_args(c, x, Wr, bias, w13_q, w2_q, ws13_q, ws2_q, out, opts);
  if (a != MOE_OK) return a;
  if (!ws_ok(workspace, workspace_bytes, fwd_layout(c).total)) return MOE_ERR_WORKSPACE;
  const Fp8Weights fw{w13_q, w13_s, w2_q, w2_s, ws13_q, ws13_s, ws2_q, ws2_s};
  return forward_fp8_impl(x, Wr, bias, fw, c, out, opts, workspace,
                          static_cast<cudaStream_t>(stream));
}

size_t moe_forward_host_workspace_bytes(const moe_cfg_t* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return fwd_layout(*cfg).total + 4 * align_up((size_t)cfg->T * cfg->H * 2);
}

int32_t moe_forward_host(const void* const* x_host, void* const* out_host, int32_t n_batches,
                         const float* Wr, const float* bias, const void* w13, const void* w2,
                         const void* ws13, const void* ws2, const moe_cfg_t* cfg, void* workspace,
                         size_t workspace_bytes, void* stream, void* h2d_stream,
                         void* d2h_stream) {
  const int32_t st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  const moe_cfg_t& c = *cfg;
  if (n_batches < 0) return MOE_ERR_INVALID_ARG;
  if (n_batches == 0 || c.T == 0) return MOE_OK;
  if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
  const size_t bytes = (size_t)c.T * c.H * 2;
  for (int b = 0; b < n_batches; ++b) {
    if (!x_host[b] || !out_host[b]) return MOE_ERR_INVALID_ARG;
    // an output must not overlap any batch's input: later batches read theirs
    // after earlier outputs have landed
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(out_host[b]);
    for (int q = 0; q < n_batches; ++q) {
      const uintptr_t x0 = reinterpret_cast<uintptr_t>(x_host[q]);
      if (o0 < x0 + bytes && x0 < o0 + bytes) return MOE_ERR_INVALID_ARG;
    }
  }
  const FwdLayout L = fwd_layout(c);
  const size_t stage = align_up(bytes);
  if (!ws_ok(workspace, workspace_bytes, L.total + 4 * stage)) return MOE_ERR_WORKSPACE;
  // staging buffers after the forward's own workspace: x of batches b % 2,
  // out of batches b % 2 (one batch computes while the next arrives and the
  // previous one leaves)
  void* xs[2] = {at<void>(workspace, L.total), at<void>(workspace, L.total + stage)};
  void* os[2] = {at<void>(workspace, L.total + 2 * stage), at<void>(workspace, L.total + 3 * stage)};
  const int32_t a = check_forward_args(c, xs[0], Wr, bias, w13, w2, ws13, ws2, os[0], nullptr);
  if (a != MOE_OK) return a;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t hs = h2d_stream ? static_cast<cudaStream_t>(h2d_stream) : s;
  cudaStream_t ds = d2h_stream ? static_cast<cudaStream_t>(d2h_stream) : s;
  // events: start, and per staging slot: input landed, forward done, output read
  struct Events {
    cudaEvent_t e[7] = {};
    ~Events() {  // released by the driver once the recorded work completes
      for (cudaEvent_t x : e)
        if (x) cudaEventDestroy(x);
    }
  } ev;
  for (cudaEvent_t& e : ev.e) RMOE_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
  cudaEvent_t start = ev.e[0], x_in[2] = {ev.e[1], ev.e[2]}, done[2] = {ev.e[3], ev.e[4]},
              o_out[2] = {ev.e[5], ev.e[6]};
  RMOE_TRY(cudaEventRecord(start, s));  // after the work already queued on stream
  RMOE_TRY(cudaStreamWaitEvent(hs, start, 0));
  RMOE_TRY(cudaStreamWaitEvent(ds, start, 0));
  for (int b = 0; b < n_batches; ++b) {
    const int k = b & 1;
    if (b >= 2) RMOE_TRY(cudaStreamWaitEvent(hs, done[k], 0));  // batch b-2 has read xs[k]
    RMOE_TRY(cudaMemcpyAsync(xs[k], x_host[b], bytes, cudaMemcpyHostToDevice, hs));
    RMOE_TRY(cudaEventRecord(x_in[k], hs));
    RMOE_TRY(cudaStreamWaitEvent(s, x_in[k], 0));
    if (b >= 2) RMOE_TRY(cudaStreamWaitEvent(s, o_out[k], 0));  // os[k] copied out
    const int32_t r = forward_impl(xs[k], Wr, bias, w13, w2, ws13, ws2, c, os[k], nullptr,
                                   workspace, b == 0, s);
    if (r != MOE_OK) return r;
    RMOE_TRY(cudaEventRecord(done[k], s));
    RMOE_TRY(cudaStreamWaitEvent(ds, done[k], 0));
    RMOE_TRY(cudaMemcpyAsync(out_host[b], os[k], bytes, cudaMemcpyDeviceToHost, ds));
    RMOE_TRY(cudaEventRecord(o_out[k], ds));
  }
  // the copies out run in order on one stream: the last one covers them all
  RMOE_TRY(cudaStreamWaitEvent(s, o_out[(n_batches - 1) & 1], 0));
  return MOE_OK;
}

size_t moe_dense_ffn_workspace_bytes(int32_t T, int32_t H, int32_t I) {
  if (T < 0 || H <= 0 || I <= 0 || H % 64 != 0 || I % 64 != 0 || H > MAX_DIM || I > MAX_DIM)
    return 0;
  // status, h [T,I], the MLP output [T,H] (added to a residual)
  return align_up(sizeof(DevStatus)) + align_up((size_t)T * I * 2) + align_up((size_t)T * H * 2);
}

int32_t moe_dense_ffn(const void* x, const void* w13, const void* w2, int32_t T, int32_t H,
                      int32_t I, const void* residual, void* out, void* workspace,
                      size_t workspace_bytes, void* stream) {
  if (T < 0 || H <= 0 || I <= 0) return MOE_ERR_INVALID_ARG;
  if (H % 64 != 0 || I % 64 != 0 || H > MAX_DIM || I > MAX_DIM) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!x || !w13 || !w2 || !out || out == x) return MOE_ERR_INVALID_ARG;
  if (!ws_ok(workspace, workspace_bytes, moe_dense_ffn_workspace_bytes(T, H, I)))
    return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = at<int>(workspace, 0);
  __nv_bfloat16* h = at<__nv_bfloat16>(workspace, align_up(sizeof(DevStatus)));
  __nv_bfloat16* y =
      at<__nv_bfloat16>(workspace, align_up(sizeof(DevStatus)) + align_up((size_t)T * I * 2));
  __nv_bfloat16* dst = residual ? y : static_cast<__nv_bfloat16*>(out);
  RMOE_TRY(launch_status_reset(status, s));
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.status = status;
  a.timeout_ns = DEFAULT_TIMEOUT_NS;
  a.alt_group = -1;
  a.single_rows = T;  // one group: every row uses the same weights
  const int sms = num_sms();
  GemmArgs up = a, down = a;
  up.k_steps = H / 64;
  up.b_second = I;
  up.out = h;
  up.ldo = I;
  up.n_valid = I;
  down.k_steps = I / 64;
  down.out = dst;
  down.ldo = H;
  down.n_valid = H;
  down.dest_mul = 1;  // output row = row
  if (T <= 64) {  // few rows: the swapped GEMMs, which stream the weights once
    const int chunk = T <= 20 ? 32 : 128;
    CUtensorMap tm_w13, tm_x, tm_w2, tm_h;
    RMOE_TRY(make_tmap_3d(&tm_w13, w13, 1, 2 * (uint64_t)I, H));
    RMOE_TRY(make_tmap_2d_box(&tm_x, x, T, H, 32));
    RMOE_TRY(make_tmap_3d(&tm_w2, w2, 1, H, I));
    RMOE_TRY(make_tmap_2d_box(&tm_h, h, T, I, 32));
    up.n_tiles = (I + 127) / 128;
    up.n_out_tile = 128;
    down.n_tiles = (H + 127) / 128;
    down.n_out_tile = 128;
    RMOE_TRY(launch_grouped_gemm_swap(EPI_SWIGLU, chunk, tm_w13, tm_x, tm_w13, tm_x, up, sms, s));
    RMOE_TRY(launch_grouped_gemm_swap(EPI_ROWSCALE, chunk, tm_w2, tm_h, tm_w2, tm_h, down, sms, s));
  } else {
    CUtensorMap tm_w13, tm_x, tm_w2, tm_h;
    RMOE_TRY(make_tmap_3d(&tm_w13, w13, 1, 2 * (uint64_t)I, H));
    RMOE_TRY(make_tmap_2d(&tm_x, x, T, H));
    RMOE_TRY(make_tmap_3d(&tm_w2, w2, 1, H, I));
    RMOE_TRY(make_tmap_2d(&tm_h, h, T, I));
    const int mt = (T + MTILE - 1) / MTILE;
    up.n_tiles = (I + 127) / 128;
    up.n_out_tile = 128;
    down.n_tiles = (H + 255) / 256;
    down.n_out_tile = 256;
    down.b_second = 128;
    RMOE_TRY(launch_grouped_gemm(EPI_SWIGLU, tm_x, tm_w13, tm_x, tm_w13, up,
                                 std::min(sms, 2 * mt * up.n_tiles), s));
    RMOE_TRY(launch_grouped_gemm(EPI_ROWSCALE, tm_h, tm_w2, tm_h, tm_w2, down,
                                 std::min(sms, 2 * mt * down.n_tiles), s));
  }
  if (residual)  // out = bf16(residual + y), fp32 sum, one rounding
    RMOE_TRY(launch_combine_slots(y, nullptr, 0, T, H, 1, residual, out, s));
  return MOE_OK;
}

int32_t moe_rows_expert_ids(const int32_t* offsets, int32_t E, int32_t R, int32_t* ids,
                            void* stream) {
  if (E <= 0 || E > MAX_E || R < 0) return MOE_ERR_INVALID_ARG;
  if (R == 0) return MOE_OK;
  if (!offsets || !ids) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_rows_expert_ids(offsets, E, R, ids, static_cast<cudaStream_t>(stream)));
}

size_t moe_expert_rows_workspace_bytes(int32_t R, int32_t H, int32_t E, int32_t I) {
  if (R < 0 || E <= 0 || E > MAX_E || H <= 0 || I <= 0 || H % 64 != 0 || I % 64 != 0 ||
      H > MAX_DIM || I > MAX_DIM)
    return 0;
  // status, the tile prefix [E+1], h [R, I]
  return align_up(sizeof(DevStatus)) + align_up((size_t)(E + 1) * 4) + align_up((size_t)R * I * 2);
}

int32_t moe_expert_rows(const void* xr, const int32_t* offsets, int32_t R, int32_t E, int32_t H,
                        int32_t I, const void* w13, const void* w2, const float* row_w,
                        const int32_t* row_dest, void* y, void* workspace, size_t workspace_bytes,
                        void* stream) {
  if (R < 0 || E <= 0 || H <= 0 || I <= 0) return MOE_ERR_INVALID_ARG;
  if (E > MAX_E || H % 64 != 0 || I % 64 != 0 || H > MAX_DIM || I > MAX_DIM)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (R == 0) return MOE_OK;
  if (!xr || !offsets || !w13 || !w2 || !row_dest || !y || y == xr) return MOE_ERR_INVALID_ARG;
  const size_t need = moe_expert_rows_workspace_bytes(R, H, E, I);
  if (!ws_ok(workspace, workspace_bytes, need)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = at<int>(workspace, 0);
  int* tiles = at<int>(workspace, align_up(sizeof(DevStatus)));
  __nv_bfloat16* h =
      at<__nv_bfloat16>(workspace, align_up(sizeof(DevStatus)) + align_up((size_t)(E + 1) * 4));
  RMOE_TRY(launch_status_reset(status, s));
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.status = status;
  a.timeout_ns = DEFAULT_TIMEOUT_NS;
  a.alt_group = -1;
  a.row_start = offsets;
  a.num_groups = E;
  GemmArgs up = a, down = a;
  up.k_steps = H / 64;
  up.b_second = I;
  up.out = h;
  up.ldo = I;
  up.n_valid = I;
  down.k_steps = I / 64;
  down.out = static_cast<__nv_bfloat16*>(y);
  down.ldo = H;
  down.n_valid = H;
  down.row_scale = row_w;
  down.dest_pos = row_dest;
  const int sms = num_sms();
  CUtensorMap tm_w13, tm_w2, tm_x, tm_h;
  RMOE_TRY(make_tmap_3d(&tm_w13, w13, E, 2 * (uint64_t)I, H));
  RMOE_TRY(make_tmap_3d(&tm_w2, w2, E, H, I));
  if ((int64_t)R <= 64LL * E) {  // few rows per expert: swapped operands
    const int chunk = (int64_t)R <= 20LL * E ? 32 : 128;
    RMOE_TRY(make_tmap_2d_box(&tm_x, xr, R, H, 32));
    RMOE_TRY(make_tmap_2d_box(&tm_h, h, R, I, 32));
    const long long chunk_bound = R / chunk + E + 1;
    up.n_tiles = (I + 127) / 128;
    up.n_out_tile = 128;
    down.n_tiles = (H + 127) / 128;
    down.n_out_tile = 128;
    RMOE_TRY(launch_grouped_gemm_swap(EPI_SWIGLU, chunk, tm_w13, tm_x, tm_w13, tm_x, up,
                                      (int)std::min<long long>(sms, chunk_bound * up.n_tiles), s));
    RMOE_TRY(launch_grouped_gemm_swap(EPI_ROWSCALE, chunk, tm_w2, tm_h, tm_w2, tm_h, down,
                                      (int)std::min<long long>(sms, chunk_bound * down.n_tiles),
                                      s));
  } else {  // 256-row tiles on CTA pairs; the tile schedule from the row offsets
    RMOE_TRY(make_tmap_2d(&tm_x, xr, R, H));
    RMOE_TRY(make_tmap_2d(&tm_h, h, R, I));
    RMOE_TRY(launch_tile_prefix(offsets, E, tiles, s));
    up.mtile_start = tiles;
    down.mtile_start = tiles;
    const long long mt_bound = R / MTILE + E;
    up.n_tiles = (I + 127) / 128;
    up.n_out_tile = 128;
    down.n_tiles = (H + 255) / 256;
    down.n_out_tile = 256;
    down.b_second = 128;
    RMOE_TRY(launch_grouped_gemm(EPI_SWIGLU, tm_x, tm_w13, tm_x, tm_w13, up,
                                 (int)std::min<long long>(sms, 2LL * mt_bound * up.n_tiles), s));
    RMOE_TRY(launch_grouped_gemm(EPI_ROWSCALE, tm_h, tm_w2, tm_h, tm_w2, down,
                                 (int)std::min<long long>(sms, 2LL * mt_bound * down.n_tiles), s));
  }
  return MOE_OK;
}

int32_t moe_combine_rows(const void* y, int32_t R, const int32_t* row_of, int32_t T, int32_t H,
                         int32_t top_k, const void* shared, const void* residual, void* out,
                         void* stream) {
  if (R < 0 || T < 0 || H <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (H % 64 != 0 || H > MAX_DIM || top_k > MAX_TOPK) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!y || !row_of || !out || out == y) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_combine_rows(y, R, row_of, top_k, T, H, shared, residual, out,
                                         static_cast<cudaStream_t>(stream)));
}

int32_t moe_rmsnorm(const void* x, const float* gamma, float eps, int32_t T, int32_t H, void* xn,
                    void* stream) {
  if (T < 0 || H <= 0 || H % 64 != 0 || H > MAX_DIM || !(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !xn) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_rmsnorm(x, gamma, eps, T, H, xn, static_cast<cudaStream_t>(stream)));
}

int32_t moe_read_device_status(void* workspace, int32_t* site, void* stream) {
  if (!workspace) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DevStatus h{0, 0};
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaMemset(workspace, 0, sizeof(h)) != cudaSuccess) return MOE_ERR_CUDA;
  if (site) *site = h.site;
  return h.code;
}

int32_t moe_selftest_wait_timeout(void* workspace, int64_t timeout_ns, void* stream) {
  if (!workspace || timeout_ns <= 0) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) % WS_ALIGN) != 0) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(workspace);
  RMOE_TRY(launch_status_reset(status, s));
  return cuda_status(launch_selftest_wait(status, (unsigned long long)timeout_ns, s));
}

}  // extern "C"
