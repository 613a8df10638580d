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
// Kernel shape: persistent, one CTA per SM (192 KB of operand stages), tiles
// of 128 rows x 256 accumulator columns, K in steps of 64 (one 128-byte
// swizzle atom).  Warp roles:
//   warp 0      one thread issues TMA tile loads into a 4-stage smem ring;
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators)
//               and one thread issues tcgen05.mma (M=128, N=256, K=16);
//   warps 2..9  epilogue: tcgen05.ld the accumulator (warp w reads TMEM
//               lanes 32*(w%4).., columns of half (w-2)/4), apply the
//               epilogue, store to global.
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

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 320;  // producer warp, MMA warp, 8 epilogue warps
constexpr int EPI_THREADS = 256;
constexpr int MAX_GROUPS = 128;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);
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
};

__device__ __forceinline__ TileCoord tile_coord(int tile, const GemmArgs& a, const int* mts,
                                                const int* rs) {
  TileCoord c;
  const int mt = tile / a.n_tiles;
  c.nt = tile - mt * a.n_tiles;
  if (a.mtile_start == nullptr) {
    c.g = 0;
    c.row0 = mt * BM;
    c.rows = min(BM, a.single_rows - c.row0);
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
  c.row0 = rs[lo] + (mt - mts[lo]) * BM;
  c.rows = min(BM, rs[lo + 1] - c.row0);
  return c;
}

__device__ __forceinline__ float silu_f(float g) { return g * __frcp_rn(1.0f + __expf(-g)); }

// One epilogue thread owns accumulator row r_in_tile and half `half` of the
// tile's columns (two warps per TMEM lane quarter).
template <int EPI>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& a, uint32_t tbase,
                                              const TileCoord& tc, int r_in_tile, int half) {
  const bool valid = r_in_tile < tc.rows;
  const int row = tc.row0 + r_in_tile;
  if constexpr (EPI == EPI_SWIGLU) {
    // accumulator columns [0,128) gate, [128,256) up; output columns nt*128 + [0,128)
    const int col0 = tc.nt * (BN / 2);
#pragma unroll 1
    for (int c = half * 64; c < half * 64 + 64; c += 32) {
      uint32_t g[32], u[32];
      tmem_ld_32x32b_x32(tbase + c, g);
      tmem_ld_32x32b_x32(tbase + BN / 2 + c, u);
      tmem_ld_wait();
      if (valid && col0 + c < a.n_valid) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float h0 = silu_f(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
          const float h1 = silu_f(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
          pk[i] = pack_bf16x2(h0, h1);
        }
        uint4* dst = reinterpret_cast<uint4*>(a.out + (size_t)row * a.ldo + col0 + c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
  } else {  // EPI_ROWSCALE: weighted rows scattered to their token-major slot
    const int col0 = tc.nt * BN;
    const float w = !valid ? 0.f : (a.row_scale ? a.row_scale[row] : 1.0f);
    const int drow = !valid ? 0 : (a.dest_pos ? a.dest_pos[row] : row * a.dest_mul + a.dest_add);
#pragma unroll 1
    for (int c = half * 128; c < half * 128 + 128; c += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tbase + c, v);
      tmem_ld_wait();
      if (valid && col0 + c < a.n_valid) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(w * __uint_as_float(v[2 * i]), w * __uint_as_float(v[2 * i + 1]));
        uint4* dst = reinterpret_cast<uint4*>(a.out + (size_t)drow * a.ldo + col0 + c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  SmemTail& st = *reinterpret_cast<SmemTail*>(smem + (size_t)STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (args.mtile_start) {
    for (int i = threadIdx.x; i <= args.num_groups; i += THREADS) {
      st.mt_start[i] = args.mtile_start[i];
      st.row_start[i] = args.row_start[i];
    }
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st.full[s], 1);
      mbar_init(&st.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st.tfull[b], 1);
      mbar_init(&st.tempty[b], EPI_THREADS);
    }
    mbar_init(&st.drain, 1);
    st.abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  __syncthreads();
  const int total_m = args.mtile_start ? st.mt_start[args.num_groups]
                                       : (args.single_rows + BM - 1) / BM;
  const int total = total_m * args.n_tiles;
  if (static_cast<int>(blockIdx.x) >= total) return;  // CTA-uniform; nothing allocated yet

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
      uint32_t armed = 0, armed_parity = 0;  // per-stage bit: armed at least once / last parity
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const TileCoord tc = tile_coord(tile, args, st.mt_start, st.row_start);
        const int nb0 = tc.nt * args.n_out_tile;
        for (int ks = 0; ks < args.k_steps; ++ks) {
          if (!mbar_wait(&st.empty[stage], phase ^ 1u, wc, 10)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + (size_t)stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          mbar_arrive_expect_tx(&st.full[stage], STAGE_BYTES);
          tma_load_2d(sa, &tmA, &st.full[stage], ks * BK, tc.row0);
          tma_load_3d(sb, &tmB, &st.full[stage], ks * BK, nb0, tc.g);
          tma_load_3d(sb + B_BYTES / 2, &tmB, &st.full[stage], ks * BK, nb0 + args.b_second,
                      tc.g);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // let every load in flight land before the CTA can exit
        for (int s = 0; s < STAGES; ++s)
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
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
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
            umma_bf16_ss(d_tmem, da + 2 * kk, db + 2 * kk, IDESC, (ks | kk) != 0 ? 1u : 0u);
          umma_commit(&st.empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&st.tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // every MMA issued by this thread completes before TMEM is released
      umma_commit(&st.drain);
      mbar_wait_drain(&st.drain, 0, args.timeout_ns);
    }
  } else {
    // ------------------------------------------------ epilogue warps 2..9
    const int q = warp & 3;           // TMEM lane quarter this warp may read
    const int half = (warp - 2) >> 2;  // which half of the tile's columns
    const int r_in_tile = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileCoord tc = tile_coord(tile, args, st.mt_start, st.row_start);
      const bool ok = mbar_wait(&st.tfull[acc], acc_phase, wc, 30);
      if (!__all_sync(FULL, ok)) break;  // warp-uniform exit
      tc_fence_after_sync();
      const uint32_t tbase =
          tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(q * 32) << 16);
      epilogue_tile<EPI>(args, tbase, tc, r_in_tile, half);
      tc_fence_before_sync();
      mbar_arrive(&st.tempty[acc]);
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
cudaError_t launch_epi(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& args,
                       int grid, cudaStream_t stream) {
  static cudaError_t attr = cudaFuncSetAttribute(
      grouped_gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (attr != cudaSuccess) return attr;
  grouped_gemm_kernel<EPI><<<grid, THREADS, SMEM_BYTES, stream>>>(tmA, tmB, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t make_tmap_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K * 2};
  const cuuint32_t box[2] = {BK, BM};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_3d(CUtensorMap* map, const void* base, uint64_t groups, uint64_t n_rows,
                         uint64_t K) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {K, n_rows, groups};
  const cuuint64_t strides[2] = {K * 2, n_rows * K * 2};
  const cuuint32_t box[3] = {BK, BN / 2, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_grouped_gemm(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB,
                                const GemmArgs& args, int grid, cudaStream_t stream) {
  if (args.mtile_start && args.num_groups > MAX_GROUPS) return cudaErrorInvalidValue;
  switch (epi) {
    case EPI_SWIGLU:
      return launch_epi<EPI_SWIGLU>(tmA, tmB, args, grid, stream);
    case EPI_ROWSCALE:
      return launch_epi<EPI_ROWSCALE>(tmA, tmB, args, grid, stream);
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
