// Router of the routed MoE block (sglang PR #32341 report, "实现拆解" step 1:
// fp32 router, sigmoid scoring + e_score_correction_bias, group-limited
// top-k, routed_scaling_factor folded in once; xxqk.cn vLLM-Omni article,
// "MoE 实现的源码级要点": selection on bias-corrected scores, gating weights
// from the raw scores, norm_topk_prob renormalisation).
//
// fp32-faithful logits on the bf16 tensor cores.  Every fp32 router weight is
// the exact sum of three bf16 terms (hi = bf16(w), mid = bf16(w - hi),
// lo = w - hi - mid: each residual has at most 16, then 8 significant bits).
// Tokens are bf16, so each product token x term is exact in fp32 and
// logits = x.hi^T + x.mid^T + x.lo^T accumulate in fp32 in TMEM -- an fp32 dot
// product of the bf16 token and the fp32 router row, up to summation order.
//   1. router_split_kernel    Wr [E,H] fp32 -> Wr3 [3,E,H] bf16
//   2. router_gemm_kernel     persistent tcgen05 GEMM over items of 128 tokens x
//                             128 experts x one K chunk; the number of chunks
//                             depends on H only (so a token's logits never
//                             depend on T); each chunk's fp32 partial goes to
//                             [S,T,E]
//   3. router_select_kernel   16 lanes per token (two tokens per warp): sums the
//                             S partials in order, then sigmoid, bias, group
//                             top-2 sums, group selection, expert selection
//                             and weights with shuffles.
#include <float.h>
#include <limits.h>

#include "common.cuh"
#include "kernels.h"

namespace rmoe {

namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int RBM = 128;  // tokens per tile
constexpr int RBN = 128;  // experts per tile (E <= 128)
constexpr int RBK = 64;
constexpr int RSTAGES = 3;
constexpr int R_A_BYTES = RBM * RBK * 2;
constexpr int R_B_BYTES = RBN * RBK * 2;
constexpr int R_STAGE_BYTES = R_A_BYTES + 3 * R_B_BYTES;
constexpr int R_THREADS = 192;
constexpr uint32_t R_TMEM_COLS = 256;  // two 128-column accumulators
constexpr int R_NP_SMALL = 32;  // expert columns per item when the batch is small
constexpr int ROUTER_WARP_SELECT_MAX_T = 4096;  // one warp per token up to this many tokens

struct __align__(8) RouterTail {
  uint64_t full[RSTAGES];
  uint64_t empty[RSTAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t R_SMEM_BYTES = 1024 + (size_t)RSTAGES * R_STAGE_BYTES + sizeof(RouterTail);

__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return;
  }
}

__global__ void __launch_bounds__(256)
    router_split_kernel(const float* __restrict__ Wr, size_t n, __nv_bfloat16* __restrict__ Wr3,
                        int* status, int clear_status, int* __restrict__ zero, int zero_n) {
  pdl_launch_dependents();
  pdl_wait();
  if (clear_status && blockIdx.x == 0 && threadIdx.x == 0) {  // first kernel of a forward
    status[0] = 0;
    status[1] = 0;
  }
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < zero_n; i += gridDim.x * blockDim.x)
    zero[i] = 0;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const float w = Wr[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);  // exact
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);  // exact, fits in bf16
    Wr3[i] = hi;
    Wr3[n + i] = mid;
    Wr3[2 * n + i] = __float2bfloat16_rn(r2);
  }
}

// Persistent: CTA b handles items b, b + gridDim.x, ... of the m_tiles x S
// items (item = token tile * S + K chunk); two TMEM accumulators let the
// epilogue of one item overlap the MMAs of the next, and the load pipeline
// runs across items.
__global__ void __launch_bounds__(R_THREADS, 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmW3, int T, int E, int k_steps,
                       int S, int NP, float* __restrict__ partial, int* status,
                       unsigned long long timeout_ns) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  RouterTail& st = *reinterpret_cast<RouterTail*>(smem + (size_t)RSTAGES * R_STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // item = (token tile, K chunk, part of NP expert columns); NP < 128 gives
  // small batches more CTAs without changing any logit's arithmetic
  const int parts = (RBN + NP - 1) / NP;
  const int items = ((T + RBM - 1) / RBM) * S * parts;
  const uint32_t idesc = idesc_bf16_f32(RBM, NP);
  const uint32_t b_bytes = (uint32_t)NP * RBK * 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < RSTAGES; ++i) {
      mbar_init(&st.full[i], 1);
      mbar_init(&st.empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st.tfull[b], 1);
      mbar_init(&st.tempty[b], 128);
    }
    mbar_init(&st.drain, 1);
    st.abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW3);
  }
  if (warp == 1) {
    tmem_alloc(&st.tmem_base, R_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = st.tmem_base;
  const WaitCtx wc{&st.abort_flag, status, timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < items; it += gridDim.x) {
        const int ms = it / parts, n0 = (it - ms * parts) * NP;
        const int m0 = (ms / S) * RBM, s = ms % S;
        const int kb = (int)((long long)s * k_steps / S);
        const int ke = (int)((long long)(s + 1) * k_steps / S);
        for (int k = kb; k < ke; ++k) {
          if (!mbar_wait(&st.empty[stage], phase ^ 1u, wc, 40)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + (size_t)stage * R_STAGE_BYTES;
          mbar_arrive_expect_tx(&st.full[stage], R_A_BYTES + 3 * b_bytes);
          tma_load_2d(sa, &tmX, &st.full[stage], k * RBK, m0);
#pragma unroll
          for (int t = 0; t < 3; ++t)
            tma_load_3d(sa + R_A_BYTES + t * R_B_BYTES, &tmW3, &st.full[stage], k * RBK, n0, t);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == RSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int i = 0; i < RSTAGES; ++i)
          if ((armed >> i) & 1u) wait_drain(&st.full[i], (armed_parity >> i) & 1u, timeout_ns);
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
      for (int it = blockIdx.x; ok && it < items; it += gridDim.x) {
        const int s = (it / parts) % S;
        const int kb = (int)((long long)s * k_steps / S);
        const int ke = (int)((long long)(s + 1) * k_steps / S);
        if (!mbar_wait(&st.tempty[acc], acc_phase ^ 1u, wc, 43)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * RBN);
        for (int k = kb; k < ke; ++k) {
          if (!mbar_wait(&st.full[stage], phase, wc, 41)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sa = smem_u32(smem + (size_t)stage * R_STAGE_BYTES);
          const uint64_t da = sdesc_kmajor_sw128(sa);
#pragma unroll
          for (int t = 0; t < 3; ++t) {
            const uint64_t db = sdesc_kmajor_sw128(sa + R_A_BYTES + t * R_B_BYTES);
#pragma unroll
            for (int kk = 0; kk < RBK / 16; ++kk)
              umma_bf16_ss(d_tmem, da + 2 * kk, db + 2 * kk, idesc,
                           (k != kb || t != 0 || kk != 0) ? 1u : 0u);
          }
          umma_commit(&st.empty[stage]);
          if (++stage == RSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&st.tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      umma_commit(&st.drain);
      wait_drain(&st.drain, 0, timeout_ns);
    }
  } else {
    // ------------------------------------------------ epilogue warps 2..5
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      const int ms = it / parts, n0 = (it - ms * parts) * NP;
      const int m0 = (ms / S) * RBM, s = ms % S;
      const bool ok = mbar_wait(&st.tfull[acc], acc_phase, wc, 42);
      if (!__all_sync(FULL, ok)) break;
      tc_fence_after_sync();
      const int row = m0 + q * 32 + lane;
      float* dst = partial + ((size_t)s * T + row) * E + n0;
      const uint32_t tbase =
          tmem_base + static_cast<uint32_t>(acc * RBN) + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < NP; c += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + c, v);
        tmem_ld_wait();
        if (row < T && n0 + c < E) {
          if (n0 + c + 32 <= E && (E & 7) == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) st_global_v8(dst + c + 8 * i, v + 8 * i);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (n0 + c + i < E) dst[c + i] = __uint_as_float(v[i]);
          }
        }
      }
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
    tmem_dealloc(tmem_base, R_TMEM_COLS);
  }
}

// Argmax over the 16 lanes of a half warp: larger value wins, equal values
// go to the lower index.
__device__ __forceinline__ void half_argmax(float& v, int& idx) {
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(FULL, v, off);
    const int oi = __shfl_xor_sync(FULL, idx, off);
    if (ov > v || (ov == v && oi < idx)) {
      v = ov;
      idx = oi;
    }
  }
}

// Two tokens per warp: lanes 0-15 take one token, lanes 16-31 the next; sub-
// lane l of a half holds experts l + 16*i (i < 8).
constexpr int SEL_WARPS = 8;
constexpr int SEL_LPT = 16;                // lanes per token
constexpr int SEL_NE = RBN / SEL_LPT;      // experts per lane

__global__ void __launch_bounds__(SEL_WARPS * 32)
    router_select_kernel(const float* __restrict__ partial, int S, const float* __restrict__ bias,
                         RouterParams p, int32_t* __restrict__ topk_ids,
                         float* __restrict__ topk_w) {
  __shared__ float sc[SEL_WARPS * 2][RBN];  // bias-corrected scores of each token
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int half = lane >> 4, sl = lane & 15;
  const int T = p.T, E = p.E;
  const int gs = E / p.n_group;
  const bool group_step = p.topk_group < p.n_group;
  float* my_sc = sc[wib * 2 + half];
  float b[SEL_NE];
  int grp[SEL_NE];
#pragma unroll
  for (int i = 0; i < SEL_NE; ++i) {
    const int e = sl + SEL_LPT * i;
    b[i] = (e < E) ? bias[e] : 0.f;
    grp[i] = (e < E) ? e / gs : 0;
  }
  const int pairs = (T + 1) / 2;
  for (int pr = blockIdx.x * SEL_WARPS + wib; pr < pairs; pr += gridDim.x * SEL_WARPS) {
    const int t = 2 * pr + half;
    const bool tok_ok = t < T;
    float s[SEL_NE], c[SEL_NE];
    bool avail[SEL_NE];
#pragma unroll
    for (int i = 0; i < SEL_NE; ++i) {
      const int e = sl + SEL_LPT * i;
      avail[i] = tok_ok && e < E;
      float l = 0.f;
      if (avail[i]) {
        l = partial[(size_t)t * E + e];
        for (int k = 1; k < S; ++k) l += partial[((size_t)k * T + t) * E + e];
      }
      s[i] = __frcp_rn(1.0f + expf(-l));  // correctly rounded: the same value as 1/(1+e^-l)
      c[i] = s[i] + b[i];
    }
    if (group_step) {
#pragma unroll
      for (int i = 0; i < SEL_NE; ++i)
        if (avail[i]) my_sc[sl + SEL_LPT * i] = c[i];
      __syncwarp();
      // sub-lane j < n_group: group score = sum of the two largest c of group j
      float G = -FLT_MAX;
      if (tok_ok && sl < p.n_group) {
        float v1 = -FLT_MAX, v2 = -FLT_MAX;
        const float* g = my_sc + sl * gs;
        for (int q = 0; q < gs; ++q) {
          const float v = g[q];
          if (v > v1) {
            v2 = v1;
            v1 = v;
          } else if (v > v2) {
            v2 = v;
          }
        }
        G = v1 + v2;
      }
      // rank of each group in its half: larger score first, ties to the lower group
      int rank = 0;
      for (int m = 0; m < p.n_group; ++m) {
        const float Gm = __shfl_sync(FULL, G, (lane & 16) | m);
        if (Gm > G || (Gm == G && m < sl)) ++rank;
      }
      const uint32_t kept =
          (__ballot_sync(FULL, sl < p.n_group && rank < p.topk_group) >> (16 * half)) & 0xFFFFu;
#pragma unroll
      for (int i = 0; i < SEL_NE; ++i)
        if (avail[i] && !((kept >> grp[i]) & 1u)) avail[i] = false;
      __syncwarp();
    }
    // top_k experts among the candidates
    int my_id = -1;
    float my_s = 0.f, sum = 0.f;
    for (int r = 0; r < p.top_k; ++r) {
      float v = -FLT_MAX;
      int idx = INT_MAX;
#pragma unroll
      for (int i = 0; i < SEL_NE; ++i) {
        const int e = sl + SEL_LPT * i;
        if (avail[i] && (c[i] > v || (c[i] == v && e < idx))) {
          v = c[i];
          idx = e;
        }
      }
      half_argmax(v, idx);
      const int owner = idx & (SEL_LPT - 1), slot = (idx >> 4) & (SEL_NE - 1);
      float sv = s[0];
#pragma unroll
      for (int i = 1; i < SEL_NE; ++i)
        if (slot == i) sv = s[i];
      sv = __shfl_sync(FULL, sv, (lane & 16) | owner);
      if (idx < E) {
        if (sl == owner) {
#pragma unroll
          for (int i = 0; i < SEL_NE; ++i)
            if (slot == i) avail[i] = false;
        }
      } else {
        sv = 0.f;
        idx = -1;  // no candidate left (non-finite scores); the permutation reports it
      }
      sum += sv;
      if (sl == r) {
        my_id = idx;
        my_s = sv;
      }
    }
    if (tok_ok && sl < p.top_k) {
      float wv = p.norm_topk_prob ? p.rsf * (my_s / sum) : p.rsf * my_s;
      if (p.mask && p.mask[t] == 0) {  // padding token: no routed expert
        my_id = -1;
        wv = 0.f;
      }
      topk_ids[(size_t)t * p.top_k + sl] = my_id;
      topk_w[(size_t)t * p.top_k + sl] = wv;
    }
  }
}

// One warp per token: lane l holds experts l + 32*i (i < 4).  The same
// arithmetic as router_select_kernel (logit sum order, sigmoid, c = s + bias,
// group score = the two largest c summed, ranking and tie rules, weights
// summed in selection order), with shorter dependency chains: every group's
// top-2 is merged across the warp by shuffles, and each selection round is one
// 4-slot scan plus a 5-level argmax.  Used for small batches (latency-bound).
__device__ __forceinline__ void warp_argmax(float& v, int& idx) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(FULL, v, off);
    const int oi = __shfl_xor_sync(FULL, idx, off);
    if (ov > v || (ov == v && oi < idx)) {
      v = ov;
      idx = oi;
    }
  }
}

constexpr int W1_NE = RBN / 32;  // expert slots per lane

__global__ void __launch_bounds__(256)
    router_select_warp_kernel(const float* __restrict__ partial, int S,
                              const float* __restrict__ bias, RouterParams p,
                              int32_t* __restrict__ topk_ids, float* __restrict__ topk_w) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int T = p.T, E = p.E;
  const int gs = E / p.n_group;
  const bool group_step = p.topk_group < p.n_group;
  float b[W1_NE];
  int gid[W1_NE];
#pragma unroll
  for (int i = 0; i < W1_NE; ++i) {
    const int e = lane + 32 * i;
    b[i] = e < E ? bias[e] : 0.f;
    gid[i] = e < E ? e / gs : -1;
  }
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    float s[W1_NE], c[W1_NE];
    uint32_t avail = 0;
#pragma unroll
    for (int i = 0; i < W1_NE; ++i) {
      const int e = lane + 32 * i;
      s[i] = 0.f;
      c[i] = -FLT_MAX;
      if (e < E) {
        float l = partial[(size_t)t * E + e];
        for (int k = 1; k < S; ++k) l += partial[((size_t)k * T + t) * E + e];
        s[i] = __frcp_rn(1.0f + expf(-l));  // correctly rounded: the same value as 1/(1+e^-l)
        c[i] = s[i] + b[i];
        avail |= 1u << i;
      }
    }
    if (group_step) {
      uint32_t kept = 0;
      float Gs[16];
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        Gs[g] = -FLT_MAX;
        if (g < p.n_group) {
          float v1 = -FLT_MAX, v2 = -FLT_MAX;  // this lane's two largest c of group g
#pragma unroll
          for (int i = 0; i < W1_NE; ++i) {
            if (gid[i] == g) {
              if (c[i] > v1) {
                v2 = v1;
                v1 = c[i];
              } else if (c[i] > v2) {
                v2 = c[i];
              }
            }
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {  // top-2 of the warp
            const float o1 = __shfl_xor_sync(FULL, v1, off);
            const float o2 = __shfl_xor_sync(FULL, v2, off);
            const float hi = fmaxf(v1, o1), lo = fminf(v1, o1);
            v2 = fmaxf(lo, fmaxf(v2, o2));
            v1 = hi;
          }
          Gs[g] = v1 + v2;
        }
      }
#pragma unroll
      for (int g = 0; g < 16; ++g) {  // larger score first, ties to the lower group
        if (g < p.n_group) {
          int rank = 0;
#pragma unroll
          for (int m = 0; m < 16; ++m)
            if (m < p.n_group && (Gs[m] > Gs[g] || (Gs[m] == Gs[g] && m < g))) ++rank;
          if (rank < p.topk_group) kept |= 1u << g;
        }
      }
#pragma unroll
      for (int i = 0; i < W1_NE; ++i)
        if (gid[i] < 0 || !((kept >> gid[i]) & 1u)) avail &= ~(1u << i);
    }
    int my_id = -1;
    float my_s = 0.f, sum = 0.f;
    for (int r = 0; r < p.top_k; ++r) {
      float v = -FLT_MAX;
      int idx = INT_MAX;
#pragma unroll
      for (int i = 0; i < W1_NE; ++i)
        if (((avail >> i) & 1u) && c[i] > v) {  // ascending ids: ties keep the lower
          v = c[i];
          idx = lane + 32 * i;
        }
      warp_argmax(v, idx);
      const int slot = (idx >> 5) & (W1_NE - 1);
      float sv = s[0];
#pragma unroll
      for (int i = 1; i < W1_NE; ++i)
        if (slot == i) sv = s[i];
      sv = __shfl_sync(FULL, sv, idx & 31);
      if (idx < E) {
        if (lane == (idx & 31)) avail &= ~(1u << slot);
      } else {
        sv = 0.f;
        idx = -1;  // no candidate left (non-finite scores); the permutation reports it
      }
      sum += sv;
      if (lane == r) {
        my_id = idx;
        my_s = sv;
      }
    }
    if (lane < p.top_k) {
      float wv = p.norm_topk_prob ? p.rsf * (my_s / sum) : p.rsf * my_s;
      if (p.mask && p.mask[t] == 0) {  // padding token: no routed expert
        my_id = -1;
        wv = 0.f;
      }
      topk_ids[(size_t)t * p.top_k + lane] = my_id;
      topk_w[(size_t)t * p.top_k + lane] = wv;
    }
  }
}

}  // namespace

int router_splits(int H) {
  const int k_steps = H / RBK;
  return k_steps / 8 > 1 ? k_steps / 8 : 1;
}

size_t router_scratch_bytes(int T, int H, int E) {
  const size_t a = ((size_t)3 * E * H * 2 + 255) & ~(size_t)255;
  return a + (size_t)router_splits(H) * T * E * 4;
}

cudaError_t launch_router(const void* x, const float* Wr, const float* bias, const RouterParams& p,
                          int32_t* topk_ids, float* topk_w, void* scratch, int* status,
                          unsigned long long timeout_ns, cudaStream_t stream) {
  const int T = p.T, H = p.H, E = p.E;
  __nv_bfloat16* Wr3 = static_cast<__nv_bfloat16*>(scratch);
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) +
                                            (((size_t)3 * E * H * 2 + 255) & ~(size_t)255));
  const size_t n = (size_t)E * H;
  const int split_grid = (int)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
  cudaError_t err = launch_chained(router_split_kernel, dim3(split_grid), dim3(256), 0, stream, Wr,
                                   n, Wr3, status, p.clear_status, p.zero, p.zero ? p.zero_n : 0);
  if (err != cudaSuccess) return err;
  const int S = router_splits(H);
  // split the expert columns when token tiles x K chunks leave most SMs idle
  const int tiles = ((T + RBM - 1) / RBM) * S;
  const int NP = tiles * (RBN / R_NP_SMALL) <= num_sms() ? R_NP_SMALL : RBN;
  CUtensorMap tmX, tmW3;
  err = make_tmap_2d(&tmX, x, (uint64_t)T, (uint64_t)H);
  if (err != cudaSuccess) return err;
  err = make_tmap_3d_box(&tmW3, Wr3, 3, (uint64_t)E, (uint64_t)H, (uint32_t)NP);
  if (err != cudaSuccess) return err;
  static std::atomic<int> smem_set[MAX_DEVICES];
  err = set_smem_limit_per_device(router_gemm_kernel, (int)R_SMEM_BYTES, smem_set);
  if (err != cudaSuccess) return err;
  const int items = tiles * (RBN / NP);
  const int grid = items < num_sms() ? items : num_sms();
  err = launch_chained(router_gemm_kernel, dim3(grid), dim3(R_THREADS), R_SMEM_BYTES, stream, tmX,
                       tmW3, T, E, H / RBK, S, NP, partial, status, timeout_ns);
  if (err != cudaSuccess) return err;
  if (T <= ROUTER_WARP_SELECT_MAX_T) {  // small batches: one warp per token, short chains
    const int grid = (T + 7) / 8;
    err = launch_chained(router_select_warp_kernel, dim3(grid), dim3(256), 0, stream,
                         (const float*)partial, S, bias, p, topk_ids, topk_w);
  } else {
    int sel_grid = ((T + 1) / 2 + SEL_WARPS - 1) / SEL_WARPS;
    const int cap = num_sms() * 16;
    if (sel_grid > cap) sel_grid = cap;
    err = launch_chained(router_select_kernel, dim3(sel_grid), dim3(SEL_WARPS * 32), 0, stream,
                         (const float*)partial, S, bias, p, topk_ids, topk_w);
  }
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace rmoe
