// Grouped expert GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The expert layers of the block (sglang PR #32341 report, "关键源码片段":
// SiLU-gated experts over packed w13 [E,2I,H] and w2 [E,H,I], router weight
// applied on the output; xxqk.cn vLLM-Omni article, "MoE 实现的源码级要点":
// bf16 grouped expert GEMMs over expert-contiguous rows, fp32 weighted
// restore, unscaled shared expert) are all D = A . B^T with
//   A  [rows, K]   bf16 rows of one group (expert) after another,
//   B  [groups, N, K] bf16 (one weight matrix per group, K-major),
// differing only in the epilogue:
//   EPI_SWIGLU   out[r, n] = bf16( silu(D[r, n]) * D[r, I + n] )   (gate|up)
//   EPI_ROWSCALE out[pos[r], n] = bf16( row_scale[r] * D[r, n] )   (router weight;
//                pos[r] = token-major slot t*(k+1)+j of row r, so that the
//                combine reads each token's slots contiguously)
//
// Kernel shape: persistent clusters of two CTAs on neighbouring SMs sharing
// one tcgen05 pair MMA (cta_group::2, M=256, N=256, K=16): a tile is 256 rows
// (128 in each CTA) x 256 accumulator columns; each CTA loads its own 128 A
// rows and its half (128 rows) of the B tile per 64-wide K step into a
// 6-stage shared-memory ring, so each SM moves 32 KB per step instead of 48.
// Warp roles (both CTAs):
//   warp 0      one thread issues TMA tile loads; their bytes are counted on
//               the leader CTA's barrier;
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulator
//               halves); in the leader one thread issues the pair MMAs and
//               commits to both CTAs' barriers;
//   warps 2..9  epilogue: tcgen05.ld the CTA's accumulator half (warp w
//               reads TMEM lanes 32*(w%4).., columns of half (w-2)/4), apply
//               the epilogue, store to global; then release the accumulator
//               on the leader's barrier.
// The epilogue of tile i overlaps the MMAs of tile i+1 (double-buffered
// accumulators).  Every wait is bounded (common.cuh): on a timeout the CTA
// records MOE_ERR_DEVICE_TIMEOUT, drains its TMA loads and MMAs, frees TMEM
// and returns.
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace rmoe {

namespace {

constexpr int BM = 128;           // rows per CTA
constexpr int TILE_M = 2 * BM;    // rows per pair tile
constexpr int BN = 256;           // accumulator columns
constexpr int BK = 64;
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;        // this CTA's A rows
constexpr int B_BYTES = (BN / 2) * BK * 2;  // this CTA's half of the B tile
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 320;  // producer warp, MMA warp, 8 epilogue warps
constexpr int EPI_THREADS = 256;
constexpr int MAX_GROUPS = 129;  // 128 experts + the shared expert
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_bf16_f32(TILE_M, BN);
constexpr int EPI_WARPS = EPI_THREADS / 32;
constexpr unsigned FULL = 0xffffffffu;

struct __align__(8) SmemTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int mt_start[MAX_GROUPS + 1];
  int row_start[MAX_GROUPS + 1];
};

constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(SmemTail);

// Wait for a phase without regard to the abort flag (used to drain work in
// flight before the CTA exits), bounded by timeout_ns.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity,
                                                uint64_t timeout_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return;
  }
}

struct TileCoord {
  int g, row0, rows, nt;
  int gstart;  // first row of the group (0 for a single group)
};

__device__ __forceinline__ TileCoord tile_coord(int tile, const GemmArgs& a, const int* mts,
                                                const int* rs) {
  TileCoord c;
  const int mt = tile / a.n_tiles;
  c.nt = tile - mt * a.n_tiles;
  if (a.mtile_start == nullptr) {
    c.g = 0;
    c.row0 = mt * TILE_M;
    c.rows = min(TILE_M, a.single_rows - c.row0);
    c.gstart = 0;
    return c;
  }
  int lo = 0, hi = a.num_groups;  // largest g with mts[g] <= mt
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (mts[mid] <= mt)
      lo = mid;
    else
      hi = mid;
  }
  c.g = lo;
  c.gstart = rs[lo];
  c.row0 = rs[lo] + (mt - mts[lo]) * TILE_M;
  c.rows = min(TILE_M, rs[lo + 1] - c.row0);
  return c;
}

// The part of a pair tile that CTA `rank` holds: rows [row0 + 128*rank, +128).
__device__ __forceinline__ TileCoord cta_part(TileCoord c, uint32_t rank) {
  c.row0 += BM * (int)rank;
  c.rows = max(0, min(BM, c.rows - BM * (int)rank));
  return c;
}

// silu(g) = g / (1 + e^-g); the same expression as in grouped_gemm_swap.cu, so
// that both kernels give the same bits.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Per-row inputs of the epilogue, read before the accumulator is waited for
// so that their latency hides behind the MMAs.
struct RowIn {
  float w;   // EPI_ROWSCALE: row weight
  int drow;  // EPI_ROWSCALE: output row
};

template <int EPI>
__device__ __forceinline__ RowIn epilogue_row_inputs(const GemmArgs& a, const TileCoord& tc,
                                                     int r_in_tile) {
  RowIn in{0.f, 0};
  if constexpr (EPI == EPI_ROWSCALE) {
    if (r_in_tile < tc.rows) {
      const int row = tc.row0 + r_in_tile;
      if (tc.g == a.alt_group || !a.dest_pos) {  // unweighted rows at t*dest_mul + dest_add
        in.w = 1.0f;
        // the group's rows are its tokens in order
        in.drow = (row - (tc.g == a.alt_group ? tc.gstart : 0)) * a.dest_mul + a.dest_add;
      } else {
        in.w = a.row_scale ? a.row_scale[row] : 1.0f;
        in.drow = a.dest_pos[row];
      }
    }
  }
  return in;
}

// One epilogue thread owns accumulator row r_in_tile and half `half` of the
// tile's columns (two warps per TMEM lane quarter).  It reads its whole half
// row into registers (back-to-back TMEM loads, one wait), hands the
// accumulator back to the MMA warp (release(): the leader's tempty barrier)
// and only then computes and stores, so that the next tiles' MMAs do not wait
// for this tile's stores.
template <int EPI, typename Release>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& a, uint32_t tbase,
                                              const TileCoord& tc, int r_in_tile, int half,
                                              const RowIn& in, Release&& release) {
  const bool valid = r_in_tile < tc.rows;
  const int row = tc.row0 + r_in_tile;
  uint32_t v[128];
  if constexpr (EPI == EPI_SWIGLU) {
    // accumulator columns [0,128) gate, [128,256) up; this half: gate and up of
    // output columns nt*128 + half*64 + [0,64), in v[0..63] and v[64..127]
    tmem_ld_32x32b_x32(tbase + half * 64, *reinterpret_cast<uint32_t(*)[32]>(v));
    tmem_ld_32x32b_x32(tbase + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
    tmem_ld_32x32b_x32(tbase + BN / 2 + half * 64, *reinterpret_cast<uint32_t(*)[32]>(v + 64));
    tmem_ld_32x32b_x32(tbase + BN / 2 + half * 64 + 32,
                       *reinterpret_cast<uint32_t(*)[32]>(v + 96));
  } else {
    // this half: accumulator columns half*128 + [0,128)
#pragma unroll
    for (int c = 0; c < 4; ++c)
      tmem_ld_32x32b_x32(tbase + half * 128 + 32 * c,
                         *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c));
  }
  tmem_ld_wait();
  release();
  if constexpr (EPI == EPI_SWIGLU) {
    const int col0 = tc.nt * (BN / 2) + half * 64;
#pragma unroll
    for (int c = 0; c < 64; c += 32) {
      if (valid && col0 + c < a.n_valid) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float h0 = silu_f(__uint_as_float(v[c + 2 * i])) * __uint_as_float(v[64 + c + 2 * i]);
          const float h1 =
              silu_f(__uint_as_float(v[c + 2 * i + 1])) * __uint_as_float(v[64 + c + 2 * i + 1]);
          pk[i] = pack_bf16x2(h0, h1);
        }
        // 64 bytes of the row as two full-sector stores
        __nv_bfloat16* dst = a.out + (size_t)row * a.ldo + col0 + c;
        st_global_v8(dst, pk);
        st_global_v8(dst + 16, pk + 8);
      }
    }
  } else {  // EPI_ROWSCALE: weighted rows scattered to their token-major slot
    const int col0 = tc.nt * BN + half * 128;
    const float w = in.w;
    const int drow = in.drow;
#pragma unroll
    for (int c = 0; c < 128; c += 32) {
      if (valid && col0 + c < a.n_valid) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(w * __uint_as_float(v[c + 2 * i]),
                              w * __uint_as_float(v[c + 2 * i + 1]));
        // 64 bytes of the row as two full-sector stores
        __nv_bfloat16* dst = a.out + (size_t)drow * a.ldo + col0 + c;
        st_global_v8(dst, pk);
        st_global_v8(dst + 16, pk + 8);
      }
    }
  }
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmA2,
                        const __grid_constant__ CUtensorMap tmB2, const GemmArgs args) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  SmemTail& st = *reinterpret_cast<SmemTail*>(smem + (size_t)STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: leader (issues the MMAs), 1: peer
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (args.mtile_start) {
    for (int i = threadIdx.x; i <= args.num_groups; i += THREADS) {
      st.mt_start[i] = args.mtile_start[i];
      st.row_start[i] = args.row_start[i];
    }
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st.full[s], 1);   // leader: its producer's expect-tx arrive
      mbar_init(&st.empty[s], 1);  // both: one commit from the leader's MMA thread
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st.tfull[b], 1);                 // both: one commit
      mbar_init(&st.tempty[b], 2 * EPI_WARPS);    // leader: every epilogue warp of both CTAs
    }
    mbar_init(&st.drain, 1);
    st.abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (args.alt_group >= 0) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB2);
    }
  }
  __syncthreads();
  const int total_m = args.mtile_start ? st.mt_start[args.num_groups]
                                       : (args.single_rows + TILE_M - 1) / TILE_M;
  const int total = total_m * args.n_tiles;
  if (cluster >= total) return;  // the same for both CTAs of the cluster; nothing allocated yet
  cluster_sync();                // both CTAs' barriers exist before any cross-CTA traffic

  if (warp == 1) {
    tmem_alloc_pair(&st.tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = st.tmem_base;
  const WaitCtx wc{&st.abort_flag, args.status, args.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // per-stage bit: armed at least once / last parity
      bool ok = true;
      for (int tile = cluster; ok && tile < total; tile += nclusters) {
        const TileCoord tc = tile_coord(tile, args, st.mt_start, st.row_start);
        const bool alt = tc.g == args.alt_group;
        // this CTA's 128 A rows at the stage's start, its half of the B tile
        // after them.  A CTA whose half of the tile holds no rows of the
        // group skips its A load (its accumulator rows are never stored); the
        // leader arms the barrier for the bytes that will actually arrive.
        const CUtensorMap* ma = alt ? &tmA2 : &tmA;
        const CUtensorMap* mb = alt ? &tmB2 : &tmB;
        const int a_row = tc.row0 + BM * (int)rank - (alt && args.alt_rebase ? tc.gstart : 0);
        const int b_grp = alt ? 0 : tc.g;
        const int b_row = tc.nt * args.n_out_tile + (int)rank * args.b_second;
        const bool load_a = tc.rows > BM * (int)rank;
        const uint32_t tx = 2 * B_BYTES + A_BYTES + (tc.rows > BM ? A_BYTES : 0);
        for (int ks = 0; ks < args.k_steps; ++ks) {
          if (!mbar_wait(&st.empty[stage], phase ^ 1u, wc, 10)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + (size_t)stage * STAGE_BYTES;
          const uint32_t full_leader = mapa_shared(smem_u32(&st.full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&st.full[stage], tx);
          if (load_a) tma_load_2d_pair(sa, ma, full_leader, ks * BK, a_row);
          tma_load_3d_pair(sa + A_BYTES, mb, full_leader, ks * BK, b_row, b_grp);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {  // both CTAs' loads are counted on the leader's barriers
        for (int s = 0; s < STAGES; ++s)
          if ((armed >> s) & 1u)
            mbar_wait_drain(&st.full[s], (armed_parity >> s) & 1u, args.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ pair MMA issuer (leader)
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total; tile += nclusters) {
        if (!mbar_wait(&st.tempty[acc], acc_phase ^ 1u, wc, 20)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int ks = 0; ks < args.k_steps; ++ks) {
          if (!mbar_wait(&st.full[stage], phase, wc, 21)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sa = smem_u32(smem + (size_t)stage * STAGE_BYTES);
          const uint64_t da = sdesc_kmajor_sw128(sa);
          const uint64_t db = sdesc_kmajor_sw128(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)  // +32 bytes along K per UMMA_K=16
            umma_bf16_ss_pair(d_tmem, da + 2 * kk, db + 2 * kk, IDESC, (ks | kk) != 0 ? 1u : 0u);
          umma_commit_pair_mask(&st.empty[stage], 0x3);  // free the stage in both CTAs
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_mask(&st.tfull[acc], 0x3);  // accumulator ready in both CTAs
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // every MMA issued by this thread completes before TMEM is released
      umma_commit_pair_mask(&st.drain, 0x1);
      mbar_wait_drain(&st.drain, 0, args.timeout_ns);
    }
  } else {
    // ------------------------------------------------ epilogue warps 2..9 (both CTAs)
    const int q = warp & 3;            // TMEM lane quarter this warp may read
    const int half = (warp - 2) >> 2;  // which half of the tile's columns
    const int r_in_tile = q * 32 + lane;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&st.tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&st.tempty[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cluster; tile < total; tile += nclusters) {
      const TileCoord tc = cta_part(tile_coord(tile, args, st.mt_start, st.row_start), rank);
      const RowIn in = epilogue_row_inputs<EPI>(args, tc, r_in_tile);
      const bool ok = mbar_wait(&st.tfull[acc], acc_phase, wc, 30);
      if (!__all_sync(FULL, ok)) break;  // warp-uniform exit
      tc_fence_after_sync();
      const uint32_t tbase =
          tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(q * 32) << 16);
      // hand the accumulator back to the leader's MMA thread
      const uint32_t tempty_leader = acc == 0 ? tempty_leader0 : tempty_leader1;
      auto release = [&]() {
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(tempty_leader);
      };
      epilogue_tile<EPI>(args, tbase, tc, r_in_tile, half, in, release);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  // both CTAs are done with both accumulators before either frees TMEM or exits
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

template <int EPI>
cudaError_t launch_epi(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmA2,
                       const CUtensorMap& tmB2, const GemmArgs& args, int grid,
                       cudaStream_t stream) {
  static std::atomic<int> smem_set[MAX_DEVICES];
  const cudaError_t attr =
      set_smem_limit_per_device(grouped_gemm_kernel<EPI>, (int)SMEM_BYTES, smem_set);
  if (attr != cudaSuccess) return attr;
  grid &= ~1;  // clusters of two CTAs
  if (grid < 2) grid = 2;
  return launch_chained(grouped_gemm_kernel<EPI>, dim3(grid), dim3(THREADS), SMEM_BYTES, stream,
                        tmA, tmB, tmA2, tmB2, args);
}

}  // namespace

cudaError_t make_tmap_2d_box(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K,
                             uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K * 2};
  const cuuint32_t box[2] = {BK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K) {
  return make_tmap_2d_box(map, base, rows, K, BM);
}

cudaError_t make_tmap_3d(CUtensorMap* map, const void* base, uint64_t groups, uint64_t n_rows,
                         uint64_t K) {
  return make_tmap_3d_box(map, base, groups, n_rows, K, BN / 2);
}

cudaError_t make_tmap_3d_box(CUtensorMap* map, const void* base, uint64_t groups,
                             uint64_t n_rows, uint64_t K, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {K, n_rows, groups};
  const cuuint64_t strides[2] = {K * 2, n_rows * K * 2};
  const cuuint32_t box[3] = {BK, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_grouped_gemm(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB,
                                const CUtensorMap& tmA2, const CUtensorMap& tmB2,
                                const GemmArgs& args, int grid, cudaStream_t stream) {
  if (args.mtile_start && args.num_groups > MAX_GROUPS) return cudaErrorInvalidValue;
  switch (epi) {
    case EPI_SWIGLU:
      return launch_epi<EPI_SWIGLU>(tmA, tmB, tmA2, tmB2, args, grid, stream);
    case EPI_ROWSCALE:
      return launch_epi<EPI_ROWSCALE>(tmA, tmB, tmA2, tmB2, args, grid, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

}  // namespace rmoe
