// Small kernels around the block: RMSNorm for a residual stack (xxqk.cn
// vLLM-Omni article, "MoE 实现的源码级要点": RMSNorm accumulates in fp32),
// the restore of the weighted expert slots, and the bounded-wait self test.
#include "common.cuh"
#include "kernels.h"

namespace rmoe {

namespace {

// One warp per row: fp32 sum of squares, xn = bf16(x * rsqrt(mean + eps) * gamma).
__global__ void __launch_bounds__(256)
    rmsnorm_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ gamma, float eps,
                   int T, int H, __nv_bfloat16* __restrict__ xn) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= T) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)row * H);
  float ss = 0.f;
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 v = src[c];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = bf16_lo(w[i]), b = bf16_hi(w[i]);
      ss = fmaf(a, a, ss);
      ss = fmaf(b, b, ss);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = rsqrtf(ss / (float)H + eps);
  uint4* dst = reinterpret_cast<uint4*>(xn + (size_t)row * H);
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 v = src[c];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a = bf16_lo(w[i]) * inv, b = bf16_hi(w[i]) * inv;
      if (gamma) {
        a *= gamma[c * 8 + 2 * i];
        b *= gamma[c * 8 + 2 * i + 1];
      }
      o[i] = pack_bf16x2(a, b);
    }
    dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Restore (xxqk.cn vLLM-Omni article, "_restore_tokens": fp32 weighted sum of
// the expert outputs): the weighted slot rows of token t sit contiguously at
// Y[t*slots .. t*slots + slots-1] (routed slots, then the shared expert), so
// one warp per token streams them with 512-byte coalesced loads and sums them
// in fp32 in slot order, then adds the residual, then rounds once.  NS: the
// slot capacity of the instantiation (slots <= NS), which sizes the per-lane
// load buffer and so the registers a thread holds.
template <int NS>
__global__ void __launch_bounds__(256, NS <= 9 ? 4 : 2)
    combine_slots_kernel(const __nv_bfloat16* __restrict__ Y, const int* __restrict__ row_of,
                         int top_k, int T, int H, int slots, int parts,
                         const __nv_bfloat16* __restrict__ residual,
                         __nv_bfloat16* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  // `parts` warps share a token (small batches), each taking every parts-th
  // 512-byte column block of the row
  for (int wt = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); wt < T * parts;
       wt += warps) {
    const int t = wt / parts, part = wt - t * parts;
    uint32_t skip = 0;  // routed slots of rejected expert ids
    for (int j = 0; j < top_k; ++j)
      if (row_of[(size_t)t * top_k + j] < 0) skip |= 1u << j;
    const uint4* src = reinterpret_cast<const uint4*>(Y + (size_t)t * slots * H);
    const int hv = H / 8;  // 16-byte vectors per row
    for (int c = lane + 32 * part; c < hv; c += 32 * parts) {
      float s[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i] = 0.f;
      uint4 y[NS];
#pragma unroll
      for (int j = 0; j < NS; ++j)
        if (j < slots) y[j] = ((skip >> j) & 1u) ? make_uint4(0, 0, 0, 0) : src[(size_t)j * hv + c];
#pragma unroll
      for (int j = 0; j < NS; ++j) {
        if (j < slots) {
          const uint32_t w[4] = {y[j].x, y[j].y, y[j].z, y[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            s[2 * i] += bf16_lo(w[i]);
            s[2 * i + 1] += bf16_hi(w[i]);
          }
        }
      }
      if (residual) {
        const uint4 v = reinterpret_cast<const uint4*>(residual + (size_t)t * H)[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          s[2 * i] += bf16_lo(w[i]);
          s[2 * i + 1] += bf16_hi(w[i]);
        }
      }
      reinterpret_cast<uint4*>(out + (size_t)t * H)[c] =
          make_uint4(pack_bf16x2(s[0], s[1]), pack_bf16x2(s[2], s[3]), pack_bf16x2(s[4], s[5]),
                     pack_bf16x2(s[6], s[7]));
    }
  }
}

__global__ void selftest_wait_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtx wc{&abort_flag, status, timeout_ns};
    (void)mbar_wait(&bar, 0, wc, 99);  // nothing arrives: must give up and report
  }
}

}  // namespace

cudaError_t launch_rmsnorm(const void* x, const float* gamma, float eps, int T, int H, void* xn,
                           cudaStream_t stream) {
  const int grid = (T + 7) / 8;
  return launch_chained(rmsnorm_kernel, dim3(grid), dim3(256), 0, stream,
                        static_cast<const __nv_bfloat16*>(x), gamma, eps, T, H,
                        static_cast<__nv_bfloat16*>(xn));
}

cudaError_t launch_combine_slots(const void* Y, const int* row_of, int top_k, int T, int H,
                                 int slots, const void* residual, void* out, cudaStream_t stream) {
  // warps per token: enough warps to fill the GPU twice over, at most one per
  // 512-byte column block of a row
  const int cap = num_sms() * 8;  // blocks of 8 warps
  int parts = (2 * cap * 8) / (T > 0 ? T : 1);
  const int max_parts = H / 256;
  if (parts > max_parts) parts = max_parts;
  if (parts < 1) parts = 1;
  long long grid = ((long long)T * parts + 7) / 8;
  if (grid > cap) grid = cap;
  auto kernel = slots <= 5 ? combine_slots_kernel<5>
               : slots <= 9 ? combine_slots_kernel<9> : combine_slots_kernel<17>;
  return launch_chained(kernel, dim3((unsigned)grid), dim3(256), 0, stream,
                        static_cast<const __nv_bfloat16*>(Y), row_of, top_k, T, H, slots, parts,
                        static_cast<const __nv_bfloat16*>(residual),
                        static_cast<__nv_bfloat16*>(out));
}

cudaError_t launch_status_reset(int* status, cudaStream_t stream) {
  return cudaMemsetAsync(status, 0, sizeof(DevStatus), stream);
}

cudaError_t launch_selftest_wait(int* status, unsigned long long timeout_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace rmoe
