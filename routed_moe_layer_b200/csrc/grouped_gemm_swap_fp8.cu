// Grouped expert GEMM with FP8 expert weights, operands swapped as in
// grouped_gemm_swap.cu (weight rows on the MMA's M = 128, an expert's token
// rows on N), for batches with few rows per expert, where the step streams
// the weights from HBM and FP8 halves those bytes.
//
// Weight format (weight-only FP8; the vLLM-Omni recipe "Robbyant/LingBot-Video",
// "Known limitations", names an FP8 backend of the upstream project without a
// format): E4M3 codes, one power-of-two scale 2^(s-127) per 128 x 128 block,
// s a UE8M0 byte.  Tokens, accumulators and outputs are as in the bf16 kernel.
//
// Dequantisation is exact.  The E4M3 byte b placed as the bf16 bit pattern
// (b & 0x80) << 8 | (b & 0x7F) << 4 is the bf16 number decode(b) * 2^-120: the
// E4M3 exponent field lands in the low four bits of the bf16 exponent field,
// E4M3 subnormals on bf16 subnormals.  One bf16 multiply by 2^(s-7) (two when
// s > 134) gives decode(b) * 2^(s-127), a bf16 value whenever it is in bf16's
// range.  The MMAs then see exactly the dequantised bf16 weights, so the result
// is bit for bit that of the bf16 kernel on those weights.
//
// Pipeline, per 128-wide K step (one scale block):
//   warp 0, one thread  TMA: the fp8 weight tile(s) [128 rows x 128 B] into a
//                       raw stage
//   warp 22, one thread TMA: the token tiles of both 64-wide K halves into a
//                       token stage (a ring of its own, so that the weight
//                       loads run as far ahead as the raw stages allow)
//   warps 6..21         per K half: dequantise the weight tile(s) into a bf16
//                       stage in the 128-byte-swizzled K-major layout of a TMA
//                       load, fence the writes to the async proxy, signal
//   warp 1, one thread  per K half: 4 UMMA_K=16 steps per weight tile
//   warps 2..5          epilogue of item i while the MMAs of item i+1 run
// A raw stage is free again as soon as the converter warps have read it, a
// token stage once the MMAs of both halves have completed: the weight ring,
// which carries the HBM stream, takes most of the shared memory and is never
// held by the MMAs.  Every wait is bounded (common.cuh).
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace rmoe {

namespace {

constexpr int WM = 128;            // weight rows per item (the MMA's M)
constexpr int BK = 64;             // K per MMA stage (one 128-byte bf16 row)
constexpr int KB8 = 128;           // K per raw stage = scale block width
constexpr int XBOX = 32;           // token rows per TMA box
constexpr int CONV_WARPS = 16;  // one 8-row swizzle atom of every weight tile each
constexpr int EPI_WARPS = 4;
constexpr int TOK_WARP = 2 + EPI_WARPS + CONV_WARPS;  // 22
constexpr int THREADS = 32 * (TOK_WARP + 1);            // 736
constexpr int MAX_GROUPS = 129;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COLS = 256;
constexpr int RAW_TILE = WM * KB8;   // fp8 weight tile: 16 KB
constexpr int W_BYTES = WM * BK * 2; // bf16 weight tile of one K half: 16 KB
constexpr int XBOX_BYTES = XBOX * BK * 2;
constexpr int MAX_RAW = 12;
constexpr int MAX_TOK = 4;
constexpr int MMA_STAGES = 2;
constexpr unsigned FULL = 0xffffffffu;

template <int EPI, int CHUNK>
struct Shape8 {
  static constexpr int NW = EPI == EPI_SWIGLU ? 2 : 1;  // weight tiles per stage
  static constexpr int X_HALF = CHUNK * BK * 2;          // token tile of one K half
  static constexpr int RAW_BYTES = NW * RAW_TILE;        // fp8 weights of one K step
  static constexpr int TOK_BYTES = 2 * X_HALF;           // tokens of one K step
  static constexpr int MMA_BYTES = NW * W_BYTES;
  static constexpr int RAW_STAGES =
      EPI == EPI_SWIGLU ? (CHUNK == 32 ? 4 : 3) : (CHUNK == 32 ? 10 : 7);
  static constexpr int TOK_STAGES = CHUNK == 32 ? 3 : 2;
  static_assert(RAW_STAGES <= MAX_RAW && TOK_STAGES <= MAX_TOK, "stage counts");
};

template <int EPI, int CHUNK>
struct __align__(8) Tail8 {
  static constexpr int TOKS = EPI == EPI_ROWSCALE ? CHUNK : 1;  // per-row epilogue inputs
  uint64_t raw_full[MAX_RAW];
  uint64_t raw_empty[MAX_RAW];
  uint64_t tok_full[MAX_TOK];
  uint64_t tok_empty[MAX_TOK];
  uint64_t mma_full[MMA_STAGES];
  uint64_t mma_empty[MMA_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int ch_start[MAX_GROUPS + 1];
  int row_start[MAX_GROUPS + 1];
  float tok_w[EPI_WARPS][TOKS];
  int tok_d[EPI_WARPS][TOKS];
};

template <int EPI, int CHUNK>
constexpr size_t smem_bytes8() {
  using S = Shape8<EPI, CHUNK>;
  return 1024 + (size_t)S::RAW_STAGES * S::RAW_BYTES + (size_t)S::TOK_STAGES * S::TOK_BYTES +
         (size_t)MMA_STAGES * S::MMA_BYTES + sizeof(Tail8<EPI, CHUNK>);
}

__device__ __forceinline__ void mbar_wait_drain8(uint64_t* bar, uint32_t parity,
                                                 uint64_t timeout_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return;
  }
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy reads (the MMAs) of the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// a * b on bf16 pairs, round to nearest even (exact here: b is a power of two);
// the -0 addend keeps the sign of a zero product.
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(0x80008000u));
  return r;
}

// The bf16 pair (m, m) with m = 2^e, -126 <= e <= 127.
__host__ __device__ constexpr uint32_t bf16x2_pow2(int e) {
  return (static_cast<uint32_t>(e + 127) << 7) * 0x00010001u;
}

struct Scale2 {
  uint32_t m1, m2;  // multipliers; m2 == 0: one multiply
};

// Multipliers that take decode(b) * 2^-120 to decode(b) * 2^(s-127).
__device__ __forceinline__ Scale2 scale_multipliers(int s) {
  Scale2 r;
  if (s <= 134) {
    r.m1 = bf16x2_pow2(s - 7);
    r.m2 = 0u;
  } else {
    r.m1 = bf16x2_pow2(127);
    r.m2 = bf16x2_pow2(s - 134);
  }
  return r;
}

// Four E4M3 codes (bytes of w, element order = byte order) to four bf16
// values: out[0] = elements 0,1, out[1] = elements 2,3.
__device__ __forceinline__ void dequant4(uint32_t w, const Scale2& sc, uint32_t* out) {
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    // byte 2p in bits 15:8, byte 2p+1 in bits 31:24, zeros elsewhere
    const uint32_t t = prmt(w, 0u, p == 0 ? 0x1404u : 0x3424u);
    // sign to bit 15 / 31, the seven magnitude bits to 10:4 / 26:20
    uint32_t v = (t & 0x80008000u) | ((t >> 4) & 0x07F007F0u);
    v = bf16x2_mul(v, sc.m1);
    if (sc.m2) v = bf16x2_mul(v, sc.m2);
    out[p] = v;
  }
}

struct Item {
  int g, row0, rows, mt;
  int gstart;
};

template <int CHUNK>
__device__ __forceinline__ Item item_coord8(int item, int n_tiles, int groups, const int* cs,
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

// The same SiLU expression as the bf16 kernels, so that the results agree bitwise.
__device__ __forceinline__ float silu_f8(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <int EPI, int CHUNK>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_swap_fp8_kernel(const __grid_constant__ CUtensorMap tmW,
                                 const __grid_constant__ CUtensorMap tmX,
                                 const __grid_constant__ CUtensorMap tmW2,
                                 const __grid_constant__ CUtensorMap tmX2, const GemmArgs args,
                                 const Fp8Scales sc) {
  using S = Shape8<EPI, CHUNK>;
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* raw_base = smem;
  uint8_t* tok_base = raw_base + (size_t)S::RAW_STAGES * S::RAW_BYTES;
  uint8_t* mma_base = tok_base + (size_t)S::TOK_STAGES * S::TOK_BYTES;
  Tail8<EPI, CHUNK>& st =
      *reinterpret_cast<Tail8<EPI, CHUNK>*>(mma_base + (size_t)MMA_STAGES * S::MMA_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int groups = args.row_start ? args.num_groups : 1;
  if (args.row_start) {
    for (int i = threadIdx.x; i <= groups; i += THREADS) st.row_start[i] = args.row_start[i];
  } else if (threadIdx.x == 0) {
    st.row_start[0] = 0;
    st.row_start[1] = args.single_rows;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S::RAW_STAGES; ++s) {
      mbar_init(&st.raw_full[s], 1);
      mbar_init(&st.raw_empty[s], CONV_WARPS);  // every converter warp has read it
    }
    for (int s = 0; s < S::TOK_STAGES; ++s) {
      mbar_init(&st.tok_full[s], 1);
      mbar_init(&st.tok_empty[s], 1);  // the MMA commit after both halves
    }
    for (int s = 0; s < MMA_STAGES; ++s) {
      mbar_init(&st.mma_full[s], CONV_WARPS);
      mbar_init(&st.mma_empty[s], 1);
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
  const int k128 = args.k_steps / 2;  // 128-wide K steps (K is a multiple of 128)

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int rs = 0;
      uint32_t rph = 0;
      uint32_t armed = 0, armed_parity = 0;  // raw stages: armed at least once / last parity
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
        const Item it =
            item_coord8<CHUNK>(item, args.n_tiles, groups, st.ch_start, st.row_start);
        const bool alt = it.g == args.alt_group;
        const CUtensorMap* mw = alt ? &tmW2 : &tmW;
        const int w_grp = alt ? 0 : it.g;
        const int w_row = it.mt * args.n_out_tile;
        for (int ks = 0; ks < k128; ++ks) {
          if (!mbar_wait(&st.raw_empty[rs], rph ^ 1u, wc, 50)) {
            ok = false;
            break;
          }
          uint8_t* sr = raw_base + (size_t)rs * S::RAW_BYTES;
          mbar_arrive_expect_tx(&st.raw_full[rs], S::NW * RAW_TILE);
          tma_load_3d(sr, mw, &st.raw_full[rs], ks * KB8, w_row, w_grp);
          if constexpr (S::NW == 2)
            tma_load_3d(sr + RAW_TILE, mw, &st.raw_full[rs], ks * KB8, args.b_second + w_row,
                        w_grp);
          armed |= 1u << rs;
          armed_parity = (armed_parity & ~(1u << rs)) | (rph << rs);
          if (++rs == S::RAW_STAGES) {
            rs = 0;
            rph ^= 1u;
          }
        }
      }
      if (!ok) {  // no TMA write may land after the CTA has exited
        for (int s = 0; s < S::RAW_STAGES; ++s)
          if ((armed >> s) & 1u)
            mbar_wait_drain8(&st.raw_full[s], (armed_parity >> s) & 1u, args.timeout_ns);
      }
    }
  } else if (warp == TOK_WARP) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer of the token tiles
      int ts = 0;
      uint32_t tph = 0;
      uint32_t armed = 0, armed_parity = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
        const Item it =
            item_coord8<CHUNK>(item, args.n_tiles, groups, st.ch_start, st.row_start);
        const bool alt = it.g == args.alt_group;
        const CUtensorMap* mx = alt ? &tmX2 : &tmX;
        const int x_row = it.row0 - (alt && args.alt_rebase ? it.gstart : 0);
        const int nb = (it.rows + XBOX - 1) / XBOX;
        const uint32_t tx = 2 * nb * XBOX_BYTES;
        for (int ks = 0; ks < k128; ++ks) {
          if (!mbar_wait(&st.tok_empty[ts], tph ^ 1u, wc, 57)) {
            ok = false;
            break;
          }
          uint8_t* sx = tok_base + (size_t)ts * S::TOK_BYTES;
          mbar_arrive_expect_tx(&st.tok_full[ts], tx);
#pragma unroll
          for (int a = 0; a < 2; ++a)
            for (int b = 0; b < nb; ++b)
              tma_load_2d(sx + a * S::X_HALF + b * XBOX_BYTES, mx, &st.tok_full[ts],
                          ks * KB8 + a * BK, x_row + b * XBOX);
          armed |= 1u << ts;
          armed_parity = (armed_parity & ~(1u << ts)) | (tph << ts);
          if (++ts == S::TOK_STAGES) {
            ts = 0;
            tph ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < S::TOK_STAGES; ++s)
          if ((armed >> s) & 1u)
            mbar_wait_drain8(&st.tok_full[s], (armed_parity >> s) & 1u, args.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int ts = 0, ms = 0;
      uint32_t tph = 0, mph = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
        const Item it =
            item_coord8<CHUNK>(item, args.n_tiles, groups, st.ch_start, st.row_start);
        const int n_pad = (it.rows + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(WM, n_pad);
        if (!mbar_wait(&st.tempty[acc], acc_phase ^ 1u, wc, 51)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * ACC_COLS;
        for (int ks = 0; ok && ks < k128; ++ks) {
          if (!mbar_wait(&st.tok_full[ts], tph, wc, 52)) {  // the token tiles
            ok = false;
            break;
          }
          const uint32_t sx = smem_u32(tok_base + (size_t)ts * S::TOK_BYTES);
#pragma unroll 1
          for (int a = 0; a < 2; ++a) {
            if (!mbar_wait(&st.mma_full[ms], mph, wc, 53)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t sw = smem_u32(mma_base + (size_t)ms * S::MMA_BYTES);
            const uint64_t dw = sdesc_kmajor_sw128(sw);
            const uint64_t dx = sdesc_kmajor_sw128(sx + a * S::X_HALF);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {  // +32 bytes along K per UMMA_K=16
              const uint32_t accum = (ks | a | kk) != 0 ? 1u : 0u;
              umma_bf16_ss(d_tmem, dw + 2 * kk, dx + 2 * kk, idesc, accum);
              if constexpr (S::NW == 2) {
                const uint64_t dw2 = sdesc_kmajor_sw128(sw + W_BYTES);
                umma_bf16_ss(d_tmem + ACC_COLS / 2, dw2 + 2 * kk, dx + 2 * kk, idesc, accum);
              }
            }
            umma_commit(&st.mma_empty[ms]);
            if (++ms == MMA_STAGES) {
              ms = 0;
              mph ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit(&st.tok_empty[ts]);  // its token tiles are read
          if (++ts == S::TOK_STAGES) {
            ts = 0;
            tph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&st.tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      umma_commit(&st.drain);  // every MMA of this thread completes before TMEM is freed
      mbar_wait_drain8(&st.drain, 0, args.timeout_ns);
    }
  } else if (warp < 2 + EPI_WARPS) {
    // ------------------------------------------------ epilogue warps 2..5
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int l = q * 32 + lane;
    const int ew = warp - 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      const Item it =
          item_coord8<CHUNK>(item, args.n_tiles, groups, st.ch_start, st.row_start);
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
      const bool ok = mbar_wait(&st.tfull[acc], acc_phase, wc, 54);
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
                const float h = silu_f8(__uint_as_float(g[j])) * __uint_as_float(u[j]);
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
  } else {
    // ------------------------------------------------ converter warps 6..21
    // Lane mapping inside one 8-row swizzle atom: lanes 8i..8i+7 take rows i and
    // i+4 (four 16-byte chunks each), so that the eight 16-byte accesses of
    // every quarter warp fall on eight different bank groups under the 128-byte
    // swizzle (chunk c of row r sits at chunk c ^ (r & 7)); the row i+4 lanes
    // store their two bf16 chunks in the opposite order for the same reason.
    const int cw = warp - 2 - EPI_WARPS;  // 0..15: rows 8cw..8cw+7 of every weight tile
    const int u = lane & 7;
    const int rr = (lane >> 3) + 4 * (u >> 2);  // row inside the atom
    const int cl = u & 3;                       // 16-byte chunk inside a K half
    const bool odd_first = (u >> 2) != 0;
    int rs = 0, ms = 0;
    uint32_t rph = 0, mph = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
      const Item it =
          item_coord8<CHUNK>(item, args.n_tiles, groups, st.ch_start, st.row_start);
      const bool alt = it.g == args.alt_group;
      const uint8_t* sexp = alt ? sc.s2 : sc.s + (size_t)it.g * sc.rows * sc.cols;
      const int w_row = it.mt * args.n_out_tile;
      // scale-block rows of the weight tiles (128-row aligned: N offsets are multiples of 128)
      const int srow0 = w_row / KB8;
      const int srow1 = (args.b_second + w_row) / KB8;
      // block scales: each K step's loaded one step ahead
      int s_next[S::NW];
      s_next[0] = __ldg(sexp + (size_t)srow0 * sc.cols);
      if constexpr (S::NW == 2) s_next[S::NW - 1] = __ldg(sexp + (size_t)srow1 * sc.cols);
      for (int ks = 0; ks < k128; ++ks) {
        Scale2 mul[S::NW];
#pragma unroll
        for (int t = 0; t < S::NW; ++t) mul[t] = scale_multipliers(s_next[t]);
        if (ks + 1 < k128) {
          s_next[0] = __ldg(sexp + (size_t)srow0 * sc.cols + ks + 1);
          if constexpr (S::NW == 2)
            s_next[S::NW - 1] = __ldg(sexp + (size_t)srow1 * sc.cols + ks + 1);
        }
        const bool got = mbar_wait(&st.raw_full[rs], rph, wc, 55);
        if (!__all_sync(FULL, got)) {
          ok = false;
          break;
        }
        const uint8_t* sr = raw_base + (size_t)rs * S::RAW_BYTES;
#pragma unroll 1
        for (int a = 0; a < 2; ++a) {
          const bool free_ = mbar_wait(&st.mma_empty[ms], mph ^ 1u, wc, 56);
          if (!__all_sync(FULL, free_)) {
            ok = false;
            break;
          }
          uint8_t* sm = mma_base + (size_t)ms * S::MMA_BYTES;
#pragma unroll
          for (int t = 0; t < S::NW; ++t) {
            {
              const int r = 8 * cw + rr;  // atom cw
              const int sw = r & 7;
              const int c = 4 * a + cl;               // fp8 chunk: K 16c..16c+15
              const uint4 v = *reinterpret_cast<const uint4*>(sr + t * RAW_TILE + r * 128 +
                                                              ((c ^ sw) << 4));
              uint32_t o[8];
              dequant4(v.x, mul[t], o + 0);
              dequant4(v.y, mul[t], o + 2);
              dequant4(v.z, mul[t], o + 4);
              dequant4(v.w, mul[t], o + 6);
              // bf16 chunks 2cl (K 16cl..+7 of this half) and 2cl+1 (K 16cl+8..+15)
              uint8_t* row = sm + t * W_BYTES + r * 128;
              const int j0 = 2 * cl;
              uint4* d0 = reinterpret_cast<uint4*>(row + ((j0 ^ sw) << 4));
              uint4* d1 = reinterpret_cast<uint4*>(row + (((j0 + 1) ^ sw) << 4));
              const uint4 lo = make_uint4(o[0], o[1], o[2], o[3]);
              const uint4 hi = make_uint4(o[4], o[5], o[6], o[7]);
              // selects, not a branch: all 32 lanes issue each of the two stores
              uint4* const first = odd_first ? d1 : d0;
              uint4* const second = odd_first ? d0 : d1;
              *first = odd_first ? hi : lo;
              *second = odd_first ? lo : hi;
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&st.mma_full[ms]);
          if (++ms == MMA_STAGES) {
            ms = 0;
            mph ^= 1u;
          }
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&st.raw_empty[rs]);  // this warp has read the weight tiles
        if (++rs == S::RAW_STAGES) {
          rs = 0;
          rph ^= 1u;
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn8() {
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

template <int EPI, int CHUNK>
cudaError_t launch_swap8(const CUtensorMap& tmW, const CUtensorMap& tmX, const CUtensorMap& tmW2,
                         const CUtensorMap& tmX2, const GemmArgs& args, const Fp8Scales& sc,
                         int grid, cudaStream_t stream) {
  constexpr size_t smem = smem_bytes8<EPI, CHUNK>();
  static_assert(smem <= 227 * 1024, "shared memory");  // 232,448 bytes per block
  static std::atomic<int> smem_set[MAX_DEVICES];
  const cudaError_t attr =
      set_smem_limit_per_device(grouped_gemm_swap_fp8_kernel<EPI, CHUNK>, (int)smem, smem_set);
  if (attr != cudaSuccess) return attr;
  if (grid < 1) grid = 1;
  return launch_chained(grouped_gemm_swap_fp8_kernel<EPI, CHUNK>, dim3(grid), dim3(THREADS), smem,
                        stream, tmW, tmX, tmW2, tmX2, args, sc);
}

}  // namespace

cudaError_t make_tmap_3d_fp8(CUtensorMap* map, const void* base, uint64_t groups, uint64_t n_rows,
                             uint64_t K) {
  auto fn = encode_fn8();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {K, n_rows, groups};
  const cuuint64_t strides[2] = {K, K * n_rows};
  const cuuint32_t box[3] = {(cuuint32_t)KB8, (cuuint32_t)WM, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_grouped_gemm_swap_fp8(int epi, int chunk, const CUtensorMap& tmW,
                                         const CUtensorMap& tmX, const CUtensorMap& tmW2,
                                         const CUtensorMap& tmX2, const GemmArgs& args,
                                         const Fp8Scales& sc, int grid, cudaStream_t stream) {
  if (args.row_start && args.num_groups > MAX_GROUPS) return cudaErrorInvalidValue;
  if (args.n_out_tile != WM || args.k_steps % 2 != 0) return cudaErrorInvalidValue;
  if (epi == EPI_SWIGLU && args.b_second % WM != 0) return cudaErrorInvalidValue;
  if (!sc.s || (args.alt_group >= 0 && !sc.s2) || sc.cols != args.k_steps / 2)
    return cudaErrorInvalidValue;
  if (epi == EPI_SWIGLU && chunk == 32)
    return launch_swap8<EPI_SWIGLU, 32>(tmW, tmX, tmW2, tmX2, args, sc, grid, stream);
  if (epi == EPI_SWIGLU && chunk == 128)
    return launch_swap8<EPI_SWIGLU, 128>(tmW, tmX, tmW2, tmX2, args, sc, grid, stream);
  if (epi == EPI_ROWSCALE && chunk == 32)
    return launch_swap8<EPI_ROWSCALE, 32>(tmW, tmX, tmW2, tmX2, args, sc, grid, stream);
  if (epi == EPI_ROWSCALE && chunk == 128)
    return launch_swap8<EPI_ROWSCALE, 128>(tmW, tmX, tmW2, tmX2, args, sc, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rmoe
