// Grouped expert GEMM for batches with few rows per expert, with the operands
// swapped ("swap AB") so that the tensor cores do not pad the tokens.
//
// The same expert layers as grouped_gemm.cu (sglang PR #32341 report,
// "关键源码片段": SiLU-gated experts over packed w13 [E,2I,H] and w2 [E,H,I],
// router weight applied on the output; xxqk.cn vLLM-Omni article,
// "MoE 实现的源码级要点": grouped expert GEMMs over expert-contiguous rows),
// computed as D^T = W . X^T: the weight rows fill the MMA's M = 128 and the
// expert's token rows its N (a multiple of 16, at most 128).  With ~15 rows per
// expert a 256-row tile would spend 94% of its tensor work on padding and
// leave the kernel bound by the MMAs instead of by streaming the weights.
//
// Work item = (chunk of at most CHUNK rows of one group, 128 weight rows):
//   EPI_SWIGLU    weight rows i0.. of the gate half and I+i0.. of the up half
//                 go to two accumulators (TMEM columns +0 and +128), so that
//                 the thread holding TMEM lane l has gate and up of output
//                 column i0+l for every token of the chunk:
//                 out[r, i0+l] = bf16( silu(gate) * up )
//   EPI_ROWSCALE  weight rows h0..h0+127 of W2: out[pos[r], h0+l] =
//                 bf16( row_scale[r] * D[l, r] )
// CHUNK is 128, or 32 when the experts hold very few rows (more of shared
// memory then goes to staging the weight stream: 6 or 10 stages instead of 4
// or 6).  Token rows come in 32-row TMA boxes (only the chunk's rows are loaded);
// weights in 128-row boxes.  Warp roles: warp 0 one thread issues the TMA
// loads; warp 1 allocates 512 TMEM columns (two accumulator buffers) and one
// thread issues the MMAs; warps 2..5 run the epilogue of item i while the MMAs
// of item i+1 proceed.  Every wait is bounded (common.cuh).
#include "common.cuh"
#include "kernels.h"

namespace rmoe {

namespace {

constexpr int WM = 128;     // weight rows per item (the MMA's M)
constexpr int BK = 64;
constexpr int XBOX = 32;    // token rows per TMA box
constexpr int THREADS = 192;
constexpr int EPI_WARPS = 4;
constexpr int MAX_GROUPS = 129;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COLS = 256;            // per accumulator buffer
constexpr int W_BYTES = WM * BK * 2;          // one weight tile
constexpr int XBOX_BYTES = XBOX * BK * 2;
constexpr int MAX_STAGES = 10;
constexpr unsigned FULL = 0xffffffffu;

// CHUNK = token rows per item (the MMA's N, padded to 16): 128, or 32 when the
// experts hold very few rows, which frees shared memory for deeper staging of
// the weight stream.
template <int EPI, int CHUNK>
struct Shape {
  static constexpr int NW = EPI == EPI_SWIGLU ? 2 : 1;  // weight tiles per stage
  static constexpr int X_BYTES = CHUNK * BK * 2;        // token tile
  static constexpr int STAGE_BYTES = NW * W_BYTES + X_BYTES;
  static constexpr int STAGES = EPI == EPI_SWIGLU ? (CHUNK == 32 ? 6 : 4) : (CHUNK == 32 ? 10 : 6);
  static_assert(STAGES <= MAX_STAGES, "stage count");
};

template <int CHUNK>
struct __align__(8) Tail {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int ch_start[MAX_GROUPS + 1];   // prefix of 128-row chunks per group
  int row_start[MAX_GROUPS + 1];  // first row of each group
  float tok_w[EPI_WARPS][CHUNK];  // EPI_ROWSCALE: each epilogue warp's copy of the
  int tok_d[EPI_WARPS][CHUNK];    //   chunk's row weights and output rows
};

template <int EPI, int CHUNK>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)Shape<EPI, CHUNK>::STAGES * Shape<EPI, CHUNK>::STAGE_BYTES +
         sizeof(Tail<CHUNK>);
}

__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity,
                                                uint64_t timeout_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return;
  }
}

struct Item {
  int g, row0, rows, mt;
  int gstart;  // first row of the group
};

template <int CHUNK>
__device__ __forceinline__ Item item_coord(int item, int n_tiles, int groups, const int* cs,
                                           const int* rs) {
  Item it;
  const int ch = item / n_tiles;
  it.mt = item - ch * n_tiles;
  int lo = 0, hi = groups;  // largest g with cs[g] <= ch (skips empty groups)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cs[mid] <= ch)
      lo = mid;
    else
      hi = mid;
  }
  it.g = lo;
  it.gstart = rs[lo];
  it.row0 = rs[lo] + (ch - cs[lo]) * CHUNK;
  it.rows = min(CHUNK, rs[lo + 1] - it.row0);
  return it;
}

// silu(g) = g / (1 + e^-g); the same expression as in grouped_gemm.cu, so that
// both kernels give the same bits.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <int EPI, int CHUNK>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmW,
                             const __grid_constant__ CUtensorMap tmX,
                             const __grid_constant__ CUtensorMap tmW2,
                             const __grid_constant__ CUtensorMap tmX2, const GemmArgs args) {
  using S = Shape<EPI, CHUNK>;
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Tail<CHUNK>& st = *reinterpret_cast<Tail<CHUNK>*>(smem + (size_t)S::STAGES * S::STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // group table: expert row offsets, or one group of single_rows rows
  const int groups = args.row_start ? args.num_groups : 1;
  if (args.row_start) {
    for (int i = threadIdx.x; i <= groups; i += THREADS) st.row_start[i] = args.row_start[i];
  } else if (threadIdx.x == 0) {
    st.row_start[0] = 0;
    st.row_start[1] = args.single_rows;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&st.full[s], 1);
      mbar_init(&st.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st.tfull[b], 1);
      mbar_init(&st.tempty[b], EPI_WARPS);
    }
    mbar_init(&st.drain, 1);
    st.abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    if (args.alt_group >= 0) {
      tma_prefetch_desc(&tmW2);
      tma_prefetch_desc(&tmX2);
    }
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefix of chunks over groups (5 groups per lane)
    constexpr int PER = (MAX_GROUPS + 31) / 32;
    int loc[PER], sum = 0;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int g = lane * PER + q;
      loc[q] = g < groups ? (st.row_start[g + 1] - st.row_start[g] + CHUNK - 1) / CHUNK : 0;
      sum += loc[q];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(FULL, incl, off);
      if (lane >= off) incl += v;
    }
    int run = incl - sum;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int g = lane * PER + q;
      if (g < groups) st.ch_start[g] = run;
      run += loc[q];
    }
    if (lane == 31) st.ch_start[groups] = incl;
  }
  __syncthreads();
  const int total = st.ch_start[groups] * args.n_tiles;
  if ((int)blockIdx.x >= total) return;  // nothing allocated yet

  if (warp == 1) {
    tmem_alloc(&st.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = st.tmem_base;
  const WaitCtx wc{&st.abort_flag, args.status, args.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
        const Item it = item_coord<CHUNK>(item, args.n_tiles, groups, st.ch_start, st.row_start);
        const bool alt = it.g == args.alt_group;
        const CUtensorMap* mw = alt ? &tmW2 : &tmW;
        const CUtensorMap* mx = alt ? &tmX2 : &tmX;
        const int w_grp = alt ? 0 : it.g;
        const int w_row = it.mt * args.n_out_tile;
        const int x_row = it.row0 - (alt && args.alt_rebase ? it.gstart : 0);
        const int nb = (it.rows + XBOX - 1) / XBOX;
        const uint32_t tx = S::NW * W_BYTES + nb * XBOX_BYTES;
        for (int ks = 0; ks < args.k_steps; ++ks) {
          if (!mbar_wait(&st.empty[stage], phase ^ 1u, wc, 40)) {
            ok = false;
            break;
          }
          uint8_t* sw = smem + (size_t)stage * S::STAGE_BYTES;
          uint8_t* sx = sw + S::NW * W_BYTES;
          mbar_arrive_expect_tx(&st.full[stage], tx);
          tma_load_3d(sw, mw, &st.full[stage], ks * BK, w_row, w_grp);
          if constexpr (S::NW == 2)
            tma_load_3d(sw + W_BYTES, mw, &st.full[stage], ks * BK, args.b_second + w_row, w_grp);
          for (int b = 0; b < nb; ++b)
            tma_load_2d(sx + b * XBOX_BYTES, mx, &st.full[stage], ks * BK, x_row + b * XBOX);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < S::STAGES; ++s)
          if ((armed >> s) & 1u)
            mbar_wait_drain(&st.full[s], (armed_parity >> s) & 1u, args.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
        const Item it = item_coord<CHUNK>(item, args.n_tiles, groups, st.ch_start, st.row_start);
        const int n_pad = (it.rows + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(WM, n_pad);
        if (!mbar_wait(&st.tempty[acc], acc_phase ^ 1u, wc, 41)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * ACC_COLS;
        for (int ks = 0; ks < args.k_steps; ++ks) {
          if (!mbar_wait(&st.full[stage], phase, wc, 42)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sw = smem_u32(smem + (size_t)stage * S::STAGE_BYTES);
          const uint64_t dw = sdesc_kmajor_sw128(sw);
          const uint64_t dx = sdesc_kmajor_sw128(sw + S::NW * W_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {  // +32 bytes along K per UMMA_K=16
            const uint32_t accum = (ks | kk) != 0 ? 1u : 0u;
            umma_bf16_ss(d_tmem, dw + 2 * kk, dx + 2 * kk, idesc, accum);
            if constexpr (S::NW == 2) {
              const uint64_t dw2 = sdesc_kmajor_sw128(sw + W_BYTES);
              umma_bf16_ss(d_tmem + ACC_COLS / 2, dw2 + 2 * kk, dx + 2 * kk, idesc, accum);
            }
          }
          umma_commit(&st.empty[stage]);
          if (++stage == S::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&st.tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      umma_commit(&st.drain);  // every MMA of this thread completes before TMEM is freed
      mbar_wait_drain(&st.drain, 0, args.timeout_ns);
    }
  } else {
    // ------------------------------------------------ epilogue warps 2..5
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int l = q * 32 + lane;
    const int ew = warp - 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      const Item it = item_coord<CHUNK>(item, args.n_tiles, groups, st.ch_start, st.row_start);
      const bool alt = it.g == args.alt_group;
      const int n_pad = (it.rows + 15) & ~15;
      const int col = it.mt * args.n_out_tile + l;  // output column of this thread
      const bool col_ok = col < args.n_valid;
      if constexpr (EPI == EPI_ROWSCALE) {  // the chunk's row weights and output rows
#pragma unroll
        for (int j = 0; j < CHUNK / 32; ++j) {
          const int n = lane + 32 * j;
          if (n < it.rows) {
            const int row = it.row0 + n;
            float w;
            int d;
            if (alt || !args.dest_pos) {
              w = 1.0f;
              d = (row - (alt ? it.gstart : 0)) * args.dest_mul + args.dest_add;
            } else {
              w = args.row_scale ? args.row_scale[row] : 1.0f;
              d = args.dest_pos[row];
            }
            st.tok_w[ew][n] = w;
            st.tok_d[ew][n] = d;
          }
        }
        __syncwarp();
      }
      const bool ok = mbar_wait(&st.tfull[acc], acc_phase, wc, 43);
      if (!__all_sync(FULL, ok)) break;  // warp-uniform exit
      tc_fence_after_sync();
      const uint32_t tb = tmem_base + static_cast<uint32_t>(acc) * ACC_COLS +
                          (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int n0 = 0; n0 < n_pad; n0 += 16) {
        if constexpr (EPI == EPI_SWIGLU) {
          uint32_t g[16], u[16];
          tmem_ld_32x32b_x16(tb + n0, g);
          tmem_ld_32x32b_x16(tb + ACC_COLS / 2 + n0, u);
          tmem_ld_wait();
          if (col_ok) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int n = n0 + j;
              if (n < it.rows) {
                const float h = silu_f(__uint_as_float(g[j])) * __uint_as_float(u[j]);
                args.out[(size_t)(it.row0 + n) * args.ldo + col] = __float2bfloat16_rn(h);
              }
            }
          }
        } else {
          uint32_t v[16];
          tmem_ld_32x32b_x16(tb + n0, v);
          tmem_ld_wait();
          if (col_ok) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int n = n0 + j;
              if (n < it.rows)
                args.out[(size_t)st.tok_d[ew][n] * args.ldo + col] =
                    __float2bfloat16_rn(st.tok_w[ew][n] * __uint_as_float(v[j]));
            }
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&st.tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int EPI, int CHUNK>
cudaError_t launch_swap(const CUtensorMap& tmW, const CUtensorMap& tmX, const CUtensorMap& tmW2,
                        const CUtensorMap& tmX2, const GemmArgs& args, int grid,
                        cudaStream_t stream) {
  constexpr size_t smem = smem_bytes<EPI, CHUNK>();
  static_assert(smem <= 227 * 1024, "shared memory");
  static std::atomic<int> smem_set[MAX_DEVICES];
  const cudaError_t attr =
      set_smem_limit_per_device(grouped_gemm_swap_kernel<EPI, CHUNK>, (int)smem, smem_set);
  if (attr != cudaSuccess) return attr;
  if (grid < 1) grid = 1;
  return launch_chained(grouped_gemm_swap_kernel<EPI, CHUNK>, dim3(grid), dim3(THREADS), smem,
                        stream, tmW, tmX, tmW2, tmX2, args);
}

}  // namespace

cudaError_t launch_grouped_gemm_swap(int epi, int chunk, const CUtensorMap& tmW,
                                     const CUtensorMap& tmX, const CUtensorMap& tmW2,
                                     const CUtensorMap& tmX2, const GemmArgs& args, int grid,
                                     cudaStream_t stream) {
  if (args.row_start && args.num_groups > MAX_GROUPS) return cudaErrorInvalidValue;
  if (args.n_out_tile != WM) return cudaErrorInvalidValue;
  if (epi == EPI_SWIGLU && chunk == 32)
    return launch_swap<EPI_SWIGLU, 32>(tmW, tmX, tmW2, tmX2, args, grid, stream);
  if (epi == EPI_SWIGLU && chunk == 128)
    return launch_swap<EPI_SWIGLU, 128>(tmW, tmX, tmW2, tmX2, args, grid, stream);
  if (epi == EPI_ROWSCALE && chunk == 32)
    return launch_swap<EPI_ROWSCALE, 32>(tmW, tmX, tmW2, tmX2, args, grid, stream);
  if (epi == EPI_ROWSCALE && chunk == 128)
    return launch_swap<EPI_ROWSCALE, 128>(tmW, tmX, tmW2, tmX2, args, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rmoe
