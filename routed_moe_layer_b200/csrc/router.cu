// Router of the routed MoE block (sglang PR #32341 report, "实现拆解" step 1:
// fp32 router, sigmoid scoring + e_score_correction_bias, group-limited
// top-k, routed_scaling_factor folded in once; xxqk.cn vLLM-Omni article,
// "MoE 实现的源码级要点": selection on bias-corrected scores, gating weights
// from the raw scores, norm_topk_prob renormalisation).
//
// One CTA scores ROUTER_TOK tokens against all experts with fp32 FMAs (x is
// exactly representable in fp32, so each logit is an fp32 dot product of the
// bf16 token and the fp32 router row), parks the logits in shared memory,
// then one warp per token does the three selections with warp shuffles.
#include <float.h>
#include <limits.h>

#include "common.cuh"
#include "kernels.h"

namespace rmoe {

namespace {

constexpr int ROUTER_TOK = 64;   // tokens per CTA
constexpr int ROUTER_EP = 128;   // expert slots per CTA (E <= 128)
constexpr int ROUTER_KC = 32;    // K chunk
constexpr int ROUTER_THREADS = 256;
constexpr int XS_LD = ROUTER_TOK + 4;
constexpr int WS_LD = ROUTER_EP + 4;
constexpr int LG_LD = ROUTER_EP + 1;
constexpr unsigned FULL = 0xffffffffu;

struct RouterSmem {
  float xs[ROUTER_KC][XS_LD];
  float ws[ROUTER_KC][WS_LD];
  float logits[ROUTER_TOK][LG_LD];
};

// Warp-wide argmax: larger value wins, equal values go to the lower index.
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

__global__ void __launch_bounds__(ROUTER_THREADS)
    router_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ Wr,
                  const float* __restrict__ bias, RouterParams p, int32_t* __restrict__ topk_ids,
                  float* __restrict__ topk_w) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  RouterSmem& sm = *reinterpret_cast<RouterSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int tok0 = blockIdx.x * ROUTER_TOK;
  const int T = p.T, H = p.H, E = p.E;

  // ---------------------------------------------------------------- logits
  const int tx = tid & 15;  // experts tx*8 .. tx*8+7
  const int ty = tid >> 4;  // tokens  ty*4 .. ty*4+3
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < H; k0 += ROUTER_KC) {
    {  // x chunk: 64 tokens x 32 k, one 8-element vector per thread
      const int t = tid >> 2, kq = tid & 3;
      const int tg = tok0 + t;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (tg < T) v = *reinterpret_cast<const uint4*>(x + (size_t)tg * H + k0 + kq * 8);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        sm.xs[kq * 8 + 2 * i][t] = bf16_lo(w4[i]);
        sm.xs[kq * 8 + 2 * i + 1][t] = bf16_hi(w4[i]);
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {  // W chunk: 128 experts x 32 k fp32
      const int f = tid + r * ROUTER_THREADS;
      const int e = f >> 3, q = f & 7;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < E) v = *reinterpret_cast<const float4*>(Wr + (size_t)e * H + k0 + q * 4);
      sm.ws[q * 4 + 0][e] = v.x;
      sm.ws[q * 4 + 1][e] = v.y;
      sm.ws[q * 4 + 2][e] = v.z;
      sm.ws[q * 4 + 3][e] = v.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < ROUTER_KC; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(&sm.xs[k][ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&sm.ws[k][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&sm.ws[k][tx * 8 + 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) sm.logits[ty * 4 + i][tx * 8 + j] = acc[i][j];
  __syncthreads();

  // ---------------------------------------------------------------- selection
  const int warp = tid >> 5, lane = tid & 31;
  const int gs = E / p.n_group;
  constexpr int NE = ROUTER_EP / 32;  // experts per lane: e = lane + 32*i
  float b[NE];
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const int e = lane + 32 * i;
    b[i] = (e < E) ? bias[e] : 0.f;
  }
  for (int tl = warp; tl < ROUTER_TOK; tl += ROUTER_THREADS / 32) {
    const int t = tok0 + tl;
    if (t >= T) break;  // warp-uniform
    float s[NE], c[NE];
    bool avail[NE];
#pragma unroll
    for (int i = 0; i < NE; ++i) {
      const int e = lane + 32 * i;
      const float l = sm.logits[tl][e < ROUTER_EP ? e : 0];
      s[i] = 1.0f / (1.0f + expf(-l));
      c[i] = s[i] + b[i];
      avail[i] = e < E;
    }
    // group-limited candidates
    if (p.topk_group < p.n_group) {
      uint32_t kept = 0;
      float G[32];
      for (int j = 0; j < p.n_group; ++j) {
        float v1 = -FLT_MAX, v2 = -FLT_MAX;
        int i1 = INT_MAX;
#pragma unroll
        for (int i = 0; i < NE; ++i) {
          const int e = lane + 32 * i;
          if (avail[i] && e / gs == j && (c[i] > v1 || (c[i] == v1 && e < i1))) {
            v1 = c[i];
            i1 = e;
          }
        }
        warp_argmax(v1, i1);
        // second best of the group: best excluding i1
#pragma unroll
        for (int i = 0; i < NE; ++i) {
          const int e = lane + 32 * i;
          if (avail[i] && e / gs == j && e != i1 && c[i] > v2) v2 = c[i];
        }
        int i2 = 0;
        warp_argmax(v2, i2);
        G[j] = v1 + v2;
      }
      for (int r = 0; r < p.topk_group; ++r) {
        int bj = -1;
        float bv = -FLT_MAX;
        for (int j = 0; j < p.n_group; ++j) {
          if (!((kept >> j) & 1u) && (bj < 0 || G[j] > bv)) {
            bv = G[j];
            bj = j;
          }
        }
        kept |= 1u << bj;
      }
#pragma unroll
      for (int i = 0; i < NE; ++i) {
        const int e = lane + 32 * i;
        if (avail[i] && !((kept >> (e / gs)) & 1u)) avail[i] = false;
      }
    }
    // top_k experts among the candidates
    int my_id = -1;
    float my_s = 0.f, sum = 0.f;
    for (int r = 0; r < p.top_k; ++r) {
      float v = -FLT_MAX;
      int idx = INT_MAX;
#pragma unroll
      for (int i = 0; i < NE; ++i) {
        const int e = lane + 32 * i;
        if (avail[i] && (c[i] > v || (c[i] == v && e < idx))) {
          v = c[i];
          idx = e;
        }
      }
      warp_argmax(v, idx);
      const int owner = idx & 31, slot = (idx >> 5) & (NE - 1);
      float sv = s[0];
#pragma unroll
      for (int i = 1; i < NE; ++i)
        if (slot == i) sv = s[i];
      sv = __shfl_sync(FULL, sv, owner);
      if (idx < E) {
        if (lane == owner) {
#pragma unroll
          for (int i = 0; i < NE; ++i)
            if (slot == i) avail[i] = false;
        }
      } else {
        sv = 0.f;
        idx = -1;  // no candidate left (non-finite scores); permute reports it
      }
      sum += sv;
      if (lane == r) {
        my_id = idx;
        my_s = sv;
      }
    }
    if (lane < p.top_k) {
      const float wv = p.norm_topk_prob ? p.rsf * (my_s / sum) : p.rsf * my_s;
      topk_ids[(size_t)t * p.top_k + lane] = my_id;
      topk_w[(size_t)t * p.top_k + lane] = wv;
    }
  }
}

}  // namespace

cudaError_t launch_router(const void* x, const float* Wr, const float* bias, const RouterParams& p,
                          int32_t* topk_ids, float* topk_w, cudaStream_t stream) {
  const int grid = (p.T + ROUTER_TOK - 1) / ROUTER_TOK;
  const size_t smem = sizeof(RouterSmem);
  cudaError_t err =
      cudaFuncSetAttribute(router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  router_kernel<<<grid, ROUTER_THREADS, smem, stream>>>(
      static_cast<const __nv_bfloat16*>(x), Wr, bias, p, topk_ids, topk_w);
  return cudaGetLastError();
}

}  // namespace rmoe
