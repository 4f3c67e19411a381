// A sampled bonus token.
//
// "Medusa no contexto de LLMs", "o que significa medusa na prática de
// deploy": after the kept branch the token the base model generates itself
// enters the sequence.  medusa_verify_accept takes its first choice; this call
// draws it instead from softmax(logits / T) at the kept node: the first token
// whose cumulative probability exceeds a uniform number from Philox4x32-10
// (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
// SC 2011), key = the 64-bit seed, counter = (64-bit offset, sequence, 0).
//
// One CTA of 1024 threads per sequence over the kept node's row: a block
// maximum, per-thread sums of exp((z - max) / T) over contiguous chunks, a
// block scan of those sums, and the thread whose interval holds u * total
// walks its chunk.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "abi_internal.h"
#include "common.cuh"

namespace medusa {

constexpr int kSampleThreads = 1024;

// first output word of Philox4x32-10 (the published round function and key
// schedule)
__device__ __forceinline__ uint32_t philox4x32_10_word0(uint32_t c0, uint32_t c1, uint32_t c2,
                                                        uint32_t c3, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c0;
}

template <typename T>
__device__ __forceinline__ float load_f(const T* p);
template <>
__device__ __forceinline__ float load_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <>
__device__ __forceinline__ float load_f<float>(const float* p) {
  return *p;
}

template <typename T>
__global__ void __launch_bounds__(kSampleThreads)
    sample_bonus_kernel(const T* __restrict__ logits, const int32_t* __restrict__ accept_len,
                        const int32_t* __restrict__ accepted_nodes, int N, int V, int width,
                        float inv_T, uint32_t seed_lo, uint32_t seed_hi, uint32_t off_lo,
                        uint32_t off_hi, int32_t* __restrict__ bonus,
                        int32_t* __restrict__ accepted_tokens, int32_t* status) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ float s_red[32];
  __shared__ int s_ired[32];
  __shared__ float s_max, s_total;
  __shared__ int s_last;
  const int b = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int L = accept_len[b];
  const int kept = (L >= 0 && L < width) ? accepted_nodes[(size_t)b * width + L] : -1;
  if (kept < 0 || kept >= N) {
    if (t == 0) report(status, MEDUSA_ERR_DEVICE_CHECK);
    return;
  }
  const T* row = logits + ((size_t)b * N + kept) * V;
  const int chunk = (V + kSampleThreads - 1) / kSampleThreads;
  const int v0 = min(V, t * chunk), v1 = min(V, v0 + chunk);
  // block maximum
  float m = -INFINITY;
  for (int v = v0; v < v1; ++v) m = fmaxf(m, load_f(row + v));
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  if (warp == 0) {
    float x = s_red[lane];
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    if (lane == 0) s_max = x;
  }
  __syncthreads();
  const float mx = s_max;
  // this chunk's sum of exp((z - max) / T)
  float s = 0.f;
  for (int v = v0; v < v1; ++v) s += expf((load_f(row + v) - mx) * inv_T);
  // block exclusive scan of the chunk sums (warp scans, then the warp totals)
  float incl = s;
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const float up = __shfl_up_sync(0xffffffffu, incl, 1);
  const float excl = lane == 0 ? 0.f : up;
  __syncthreads();
  if (lane == 31) s_red[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const float wsum = s_red[lane];
    float wincl = wsum;
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += y;
    }
    const float wup = __shfl_up_sync(0xffffffffu, wincl, 1);
    s_red[lane] = lane == 0 ? 0.f : wup;  // exclusive prefix of the warp totals
    if (lane == 31) s_total = wincl;
  }
  __syncthreads();
  const float prefix = s_red[warp] + excl;
  const uint32_t x = philox4x32_10_word0(off_lo, off_hi, (uint32_t)b, 0u, seed_lo, seed_hi);
  const float target = (float)(x >> 8) * 5.9604644775390625e-8f * s_total;  // u * total
  // the walking thread: the last chunk with mass whose prefix is <= target
  // (one thread by construction, whatever the rounding of the scan)
  int cand = (s > 0.f && prefix <= target) ? t : -1;
  for (int o = 16; o > 0; o >>= 1) cand = max(cand, __shfl_xor_sync(0xffffffffu, cand, o));
  if (lane == 0) s_ired[warp] = cand;
  __syncthreads();
  if (warp == 0) {
    int c2 = s_ired[lane];
    for (int o = 16; o > 0; o >>= 1) c2 = max(c2, __shfl_xor_sync(0xffffffffu, c2, o));
    if (lane == 0) s_last = c2;
  }
  __syncthreads();
  if (s_last < 0) {  // no mass anywhere: a NaN in the row
    if (t == 0) report(status, MEDUSA_ERR_DEVICE_CHECK);
    return;
  }
  if (t == s_last) {
    int tok = v1 - 1;
    float acc = prefix;
    for (int v = v0; v < v1; ++v) {
      const float w = expf((load_f(row + v) - mx) * inv_T);
      acc += w;
      if (w > 0.f) tok = v;
      if (acc > target && w > 0.f) break;
    }
    bonus[b] = tok;
    accepted_tokens[(size_t)b * width + L] = tok;
  }
}

medusa_status_t sample_bonus(const void* logits, medusa_dtype_t dt, const int32_t* accept_len,
                             const int32_t* accepted_nodes, int B, int N, int V, int max_depth,
                             float temperature, uint64_t seed, uint64_t offset, int32_t* bonus,
                             int32_t* accepted_tokens, int32_t* status, cudaStream_t stream) {
  const float inv_T = 1.0f / temperature;
  const uint32_t s0 = (uint32_t)seed, s1 = (uint32_t)(seed >> 32);
  const uint32_t o0 = (uint32_t)offset, o1 = (uint32_t)(offset >> 32);
  if (dt == MEDUSA_BF16)
    launch(sample_bonus_kernel<__nv_bfloat16>, B, kSampleThreads, 0, stream,
           static_cast<const __nv_bfloat16*>(logits), accept_len, accepted_nodes, N, V,
           max_depth + 1, inv_T, s0, s1, o0, o1, bonus, accepted_tokens, status);
  else
    launch(sample_bonus_kernel<float>, B, kSampleThreads, 0, stream,
           static_cast<const float*>(logits), accept_len, accepted_nodes, N, V, max_depth + 1,
           inv_T, s0, s1, o0, o1, bonus, accepted_tokens, status);
  return check_launch("sample_bonus");
}

}  // namespace medusa
