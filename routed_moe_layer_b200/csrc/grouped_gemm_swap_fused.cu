// Both expert projections of a small batch in one persistent launch, with
// swapped operands as in grouped_gemm_swap.cu (weight rows on the MMA's
// M = 128, a chunk of an expert's rows on N): the expert layers of the block
// (sglang PR #32341 report, "关键源码片段": SiLU-gated experts over packed w13
// [E,2I,H] and w2 [E,H,I], router weight applied on the output; xxqk.cn
// vLLM-Omni article, "MoE 实现的源码级要点": grouped expert GEMMs over
// expert-contiguous rows, unscaled shared expert as one more group).
//
// With few rows per expert the step streams the expert weights from HBM, and
// two launches leave each one's last wave of items half empty and put a ramp
// between them.  Here the work items of both projections form one sequence:
//   items [0, U)      up:   (chunk, 128 h columns): h = silu(x.Wg^T) * (x.Wu^T)
//   items [U, U + D)  down: (chunk, 128 output columns): Y[pos] = w * (h.W2^T)
// claimed one at a time from a global counter, so every up item is claimed
// (by a running CTA) before any down item.  A down item reads the h rows of
// its chunk, which the chunk's up items write: each up item's four epilogue
// warps add 1 to the chunk's ready counter after storing (release at GPU
// scope), and the TMA thread of a down item waits (bounded, acquire) for
// 4 * (up items per chunk) before loading those rows through the async proxy.
// The waits therefore only ever wait on items held by running CTAs.
//
// Each item's arithmetic is exactly that of grouped_gemm_swap.cu (the same MMA
// shapes, K order and epilogue expressions), so the results are the same bits.
//
// Shared-memory stage: two 16 KB weight tiles and two token tiles.  An up item
// uses one stage per 64-wide K step (gate tile, up tile, its rows); a down item
// two K steps per stage (two weight tiles, two h tiles).
// Warp roles: warp 0 one thread claims items and issues the TMA loads; warp 1
// allocates TMEM (two 256-column accumulator buffers) and one thread issues
// the MMAs; warps 2..5 run the epilogues.  Every wait is bounded (common.cuh).
#include "common.cuh"
#include "kernels.h"

namespace rmoe {

namespace {

constexpr int WM = 128;
constexpr int BK = 64;
constexpr int XBOX = 32;
constexpr int THREADS = 192;
constexpr int EPI_WARPS = 4;
constexpr int MAX_GROUPS = 129;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COLS = 256;
constexpr int W_BYTES = WM * BK * 2;
constexpr int XBOX_BYTES = XBOX * BK * 2;
constexpr int MAX_STAGES = 5;
constexpr int RING = 4;  // claimed items handed from the TMA thread to the other roles
constexpr unsigned FULL = 0xffffffffu;

template <int CHUNK>
struct FShape {
  static constexpr int X_BYTES = CHUNK * BK * 2;
  static constexpr int STAGE_BYTES = 2 * W_BYTES + 2 * X_BYTES;
  static constexpr int STAGES = CHUNK == 32 ? 5 : 3;
  static_assert(STAGES <= MAX_STAGES, "stage count");
};

template <int CHUNK>
struct __align__(8) FTail {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t item_full[RING];
  uint64_t item_empty[RING];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int items[RING];
  int ch_start[MAX_GROUPS + 1];
  int row_start[MAX_GROUPS + 1];
  float tok_w[EPI_WARPS][CHUNK];
  int tok_d[EPI_WARPS][CHUNK];
};

template <int CHUNK>
constexpr size_t fsmem_bytes() {
  return 1024 + (size_t)FShape<CHUNK>::STAGES * FShape<CHUNK>::STAGE_BYTES +
         sizeof(FTail<CHUNK>);
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return;
  }
}

struct FItem {
  bool down;
  int g, row0, rows, mt, gstart, ch;
};

template <int CHUNK>
__device__ __forceinline__ FItem fitem(int item, int U, int n_up, int n_down, int groups,
                                       const int* cs, const int* rs) {
  FItem it;
  int ch;
  if (item < U) {
    it.down = false;
    ch = item / n_up;
    it.mt = item - ch * n_up;
  } else {
    it.down = true;
    const int j = item - U;
    ch = j / n_down;
    it.mt = j - ch * n_down;
  }
  int lo = 0, hi = groups;  // largest g with cs[g] <= ch (skips empty groups)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cs[mid] <= ch)
      lo = mid;
    else
      hi = mid;
  }
  it.ch = ch;
  it.g = lo;
  it.gstart = rs[lo];
  it.row0 = rs[lo] + (ch - cs[lo]) * CHUNK;
  it.rows = min(CHUNK, rs[lo + 1] - it.row0);
  return it;
}

// silu(g) = g / (1 + e^-g): the expression of the other GEMM kernels, so that
// all of them give the same bits.
__device__ __forceinline__ float silu_x(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// The next claimed item from the ring (-1: none left); every consumer role
// reads each item once, in the same order.
__device__ __forceinline__ int next_item(uint64_t* full, const int* items, int slot,
                                         uint32_t phase, const WaitCtx& wc, int site, bool& ok) {
  if (!mbar_wait(&full[slot], phase, wc, site)) {
    ok = false;
    return -1;
  }
  return items[slot];
}

template <int CHUNK>
__global__ void __launch_bounds__(THREADS, 1)
    swap_fused_kernel(const __grid_constant__ CUtensorMap tmW13,
                      const __grid_constant__ CUtensorMap tmXp,
                      const __grid_constant__ CUtensorMap tmWs13,
                      const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmW2,
                      const __grid_constant__ CUtensorMap tmH,
                      const __grid_constant__ CUtensorMap tmWs2, const GemmArgs up,
                      const GemmArgs dn, int* sched) {
  using S = FShape<CHUNK>;
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  FTail<CHUNK>& st = *reinterpret_cast<FTail<CHUNK>*>(smem + (size_t)S::STAGES * S::STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* claim = sched;      // next unclaimed item
  int* ready = sched + 1;  // per chunk: up-item epilogue warps done

  const int groups = up.num_groups;
  for (int i = threadIdx.x; i <= groups; i += THREADS) st.row_start[i] = up.row_start[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&st.full[s], 1);
      mbar_init(&st.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st.tfull[b], 1);
      mbar_init(&st.tempty[b], EPI_WARPS);
    }
    for (int r = 0; r < RING; ++r) {
      mbar_init(&st.item_full[r], 1);
      mbar_init(&st.item_empty[r], 1 + EPI_WARPS);  // the MMA thread + each epilogue warp
    }
    mbar_init(&st.drain, 1);
    st.abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmW13);
    tma_prefetch_desc(&tmXp);
    tma_prefetch_desc(&tmW2);
    tma_prefetch_desc(&tmH);
    if (up.alt_group >= 0) {
      tma_prefetch_desc(&tmWs13);
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmWs2);
    }
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefix of chunks over groups
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
  const int chunks = st.ch_start[groups];
  const int U = chunks * up.n_tiles;
  const int total = U + chunks * dn.n_tiles;

  if (warp == 1) {
    tmem_alloc(&st.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = st.tmem_base;
  const WaitCtx wc{&st.abort_flag, up.status, up.timeout_ns};
  const int ready_target = EPI_WARPS * up.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ claims + TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      int rslot = 0;
      uint32_t rphase = 0;
      bool ok = true;
      int item = atomicAdd(claim, 1);
      for (;;) {
        // hand the item (or the end, -1) to the MMA thread and the epilogue warps
        if (!mbar_wait(&st.item_empty[rslot], rphase ^ 1u, wc, 60)) {
          ok = false;
          break;
        }
        const bool last = item >= total;
        st.items[rslot] = last ? -1 : item;
        mbar_arrive(&st.item_full[rslot]);
        if (++rslot == RING) {
          rslot = 0;
          rphase ^= 1u;
        }
        if (last) break;
        const int next = atomicAdd(claim, 1);  // its latency hides behind this item's loads
        const FItem it = fitem<CHUNK>(item, U, up.n_tiles, dn.n_tiles, groups, st.ch_start,
                                      st.row_start);
        const GemmArgs& a = it.down ? dn : up;
        const bool alt = it.g == a.alt_group;
        const int w_grp = alt ? 0 : it.g;
        const int w_row = it.mt * a.n_out_tile;
        const int nb = (it.rows + XBOX - 1) / XBOX;
        if (!it.down) {
          const CUtensorMap* mw = alt ? &tmWs13 : &tmW13;
          const CUtensorMap* mx = alt ? &tmX : &tmXp;
          const int x_row = it.row0 - (alt ? it.gstart : 0);  // the shared group reads x
          const uint32_t tx = 2 * W_BYTES + nb * XBOX_BYTES;
          for (int ks = 0; ks < a.k_steps; ++ks) {
            if (!mbar_wait(&st.empty[stage], phase ^ 1u, wc, 61)) {
              ok = false;
              break;
            }
            uint8_t* sw = smem + (size_t)stage * S::STAGE_BYTES;
            uint8_t* sx = sw + 2 * W_BYTES;
            mbar_arrive_expect_tx(&st.full[stage], tx);
            tma_load_3d(sw, mw, &st.full[stage], ks * BK, w_row, w_grp);
            tma_load_3d(sw + W_BYTES, mw, &st.full[stage], ks * BK, a.b_second + w_row, w_grp);
            for (int b = 0; b < nb; ++b)
              tma_load_2d(sx + b * XBOX_BYTES, mx, &st.full[stage], ks * BK, x_row + b * XBOX);
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == S::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        } else {
          // the chunk's h rows: written by its up items on this and other SMs
          const uint64_t t0 = globaltimer_ns();
          for (;;) {
            int v;
            asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ready + it.ch)
                         : "memory");
            if (v >= ready_target) break;
            if (*wc.abort_flag) {
              ok = false;
              break;
            }
            if (globaltimer_ns() - t0 > wc.timeout_ns) {
              *wc.abort_flag = 1;
              report_error(wc.status, MOE_ERR_DEVICE_TIMEOUT, 62);
              ok = false;
              break;
            }
          }
          if (!ok) break;
          asm volatile("fence.proxy.async.global;" ::: "memory");  // generic writes -> TMA reads
          const CUtensorMap* mw = alt ? &tmWs2 : &tmW2;
          const int x_row = it.row0;  // h rows, shared group included, where they are
          for (int ks = 0; ks < a.k_steps; ks += 2) {
            const int nk = min(2, a.k_steps - ks);
            if (!mbar_wait(&st.empty[stage], phase ^ 1u, wc, 63)) {
              ok = false;
              break;
            }
            uint8_t* sw = smem + (size_t)stage * S::STAGE_BYTES;
            uint8_t* sx = sw + 2 * W_BYTES;
            mbar_arrive_expect_tx(&st.full[stage], nk * (W_BYTES + nb * XBOX_BYTES));
            for (int h = 0; h < nk; ++h) {
              tma_load_3d(sw + h * W_BYTES, mw, &st.full[stage], (ks + h) * BK, w_row, w_grp);
              for (int b = 0; b < nb; ++b)
                tma_load_2d(sx + h * S::X_BYTES + b * XBOX_BYTES, &tmH, &st.full[stage],
                            (ks + h) * BK, x_row + b * XBOX);
            }
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == S::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) break;
        item = next;
      }
      if (!ok) {  // no TMA write may land after the CTA has exited
        for (int s = 0; s < S::STAGES; ++s)
          if ((armed >> s) & 1u) drain_wait(&st.full[s], (armed_parity >> s) & 1u, up.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      int rslot = 0;
      uint32_t rphase = 0;
      bool ok = true;
      for (;;) {
        const int item = next_item(st.item_full, st.items, rslot, rphase, wc, 64, ok);
        if (!ok) break;
        mbar_arrive(&st.item_empty[rslot]);
        if (++rslot == RING) {
          rslot = 0;
          rphase ^= 1u;
        }
        if (item < 0) break;
        const FItem it = fitem<CHUNK>(item, U, up.n_tiles, dn.n_tiles, groups, st.ch_start,
                                      st.row_start);
        const int k_steps = it.down ? dn.k_steps : up.k_steps;
        const int n_pad = (it.rows + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(WM, n_pad);
        if (!mbar_wait(&st.tempty[acc], acc_phase ^ 1u, wc, 65)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * ACC_COLS;
        const int kstep_per_stage = it.down ? 2 : 1;
        for (int ks = 0; ok && ks < k_steps; ks += kstep_per_stage) {
          if (!mbar_wait(&st.full[stage], phase, wc, 66)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sw = smem_u32(smem + (size_t)stage * S::STAGE_BYTES);
          if (!it.down) {
            const uint64_t dw = sdesc_kmajor_sw128(sw);
            const uint64_t dw2 = sdesc_kmajor_sw128(sw + W_BYTES);
            const uint64_t dx = sdesc_kmajor_sw128(sw + 2 * W_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {  // +32 bytes along K per UMMA_K=16
              const uint32_t accum = (ks | kk) != 0 ? 1u : 0u;
              umma_bf16_ss(d_tmem, dw + 2 * kk, dx + 2 * kk, idesc, accum);
              umma_bf16_ss(d_tmem + ACC_COLS / 2, dw2 + 2 * kk, dx + 2 * kk, idesc, accum);
            }
          } else {
            const int nk = min(2, k_steps - ks);
            for (int h = 0; h < nk; ++h) {
              const uint64_t dw = sdesc_kmajor_sw128(sw + h * W_BYTES);
              const uint64_t dx = sdesc_kmajor_sw128(sw + 2 * W_BYTES + h * S::X_BYTES);
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk) {
                const uint32_t accum = ((ks + h) | kk) != 0 ? 1u : 0u;
                umma_bf16_ss(d_tmem, dw + 2 * kk, dx + 2 * kk, idesc, accum);
              }
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
      drain_wait(&st.drain, 0, up.timeout_ns);
    }
  } else {
    // ------------------------------------------------ epilogue warps 2..5
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int l = q * 32 + lane;
    const int ew = warp - 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    int rslot = 0;
    uint32_t rphase = 0;
    bool ok = true;
    for (;;) {
      const int item = next_item(st.item_full, st.items, rslot, rphase, wc, 67, ok);
      if (!__all_sync(FULL, ok)) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&st.item_empty[rslot]);
      if (++rslot == RING) {
        rslot = 0;
        rphase ^= 1u;
      }
      if (item < 0) break;
      const FItem it = fitem<CHUNK>(item, U, up.n_tiles, dn.n_tiles, groups, st.ch_start,
                                    st.row_start);
      const GemmArgs& a = it.down ? dn : up;
      const bool alt = it.g == a.alt_group;
      const int n_pad = (it.rows + 15) & ~15;
      const int col = it.mt * a.n_out_tile + l;  // output column of this thread
      const bool col_ok = col < a.n_valid;
      if (it.down) {  // the chunk's row weights and output rows
#pragma unroll
        for (int j = 0; j < CHUNK / 32; ++j) {
          const int n = lane + 32 * j;
          if (n < it.rows) {
            const int row = it.row0 + n;
            float w;
            int d;
            if (alt || !a.dest_pos) {
              w = 1.0f;
              d = (row - (alt ? it.gstart : 0)) * a.dest_mul + a.dest_add;
            } else {
              w = a.row_scale ? a.row_scale[row] : 1.0f;
              d = a.dest_pos[row];
            }
            st.tok_w[ew][n] = w;
            st.tok_d[ew][n] = d;
          }
        }
        __syncwarp();
      }
      const bool got = mbar_wait(&st.tfull[acc], acc_phase, wc, 68);
      if (!__all_sync(FULL, got)) break;  // warp-uniform exit
      tc_fence_after_sync();
      const uint32_t tb = tmem_base + static_cast<uint32_t>(acc) * ACC_COLS +
                          (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int n0 = 0; n0 < n_pad; n0 += 16) {
        if (!it.down) {
          uint32_t g[16], u[16];
          tmem_ld_32x32b_x16(tb + n0, g);
          tmem_ld_32x32b_x16(tb + ACC_COLS / 2 + n0, u);
          tmem_ld_wait();
          if (col_ok) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int n = n0 + j;
              if (n < it.rows) {
                const float h = silu_x(__uint_as_float(g[j])) * __uint_as_float(u[j]);
                a.out[(size_t)(it.row0 + n) * a.ldo + col] = __float2bfloat16_rn(h);
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
                a.out[(size_t)st.tok_d[ew][n] * a.ldo + col] =
                    __float2bfloat16_rn(st.tok_w[ew][n] * __uint_as_float(v[j]));
            }
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&st.tempty[acc]);
      if (!it.down) {  // the chunk's h columns of this warp are stored: count them
        asm volatile("fence.acq_rel.gpu;" ::: "memory");
        __syncwarp();
        if (lane == 0) atomicAdd(ready + it.ch, 1);
      }
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

template <int CHUNK>
cudaError_t launch_fused(const CUtensorMap* maps, const GemmArgs& up, const GemmArgs& dn,
                         int* sched, int grid, cudaStream_t stream) {
  constexpr size_t smem = fsmem_bytes<CHUNK>();
  static_assert(smem <= 227 * 1024, "shared memory");
  static std::atomic<int> smem_set[MAX_DEVICES];
  const cudaError_t attr = set_smem_limit_per_device(swap_fused_kernel<CHUNK>, (int)smem, smem_set);
  if (attr != cudaSuccess) return attr;
  if (grid < 1) grid = 1;
  return launch_chained(swap_fused_kernel<CHUNK>, dim3(grid), dim3(THREADS), smem, stream,
                        maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], up, dn,
                        sched);
}

}  // namespace

cudaError_t launch_swap_fused(int chunk, const CUtensorMap* maps, const GemmArgs& up,
                              const GemmArgs& dn, int* sched, int grid, cudaStream_t stream) {
  if (!up.row_start || up.num_groups > MAX_GROUPS || up.num_groups != dn.num_groups)
    return cudaErrorInvalidValue;
  if (up.n_out_tile != WM || dn.n_out_tile != WM) return cudaErrorInvalidValue;
  if (chunk == 32) return launch_fused<32>(maps, up, dn, sched, grid, stream);
  if (chunk == 128) return launch_fused<128>(maps, up, dn, sched, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rmoe
