// Verification and acceptance of the candidate tree.
//
// "Medusa Heads" glossary, "Attention arborescente et acceptation": the
// longest branch the model agrees with is kept.  Greedy: a candidate is
// accepted when it equals the model's first choice.  Typical: a candidate is
// kept when its base-model probability exceeds a threshold tied to the
// entropy of the distribution, here min(eps, delta * exp(-H)).
// "Medusa no contexto de LLMs": on rejection the model's own token is used.
//
// Two launches.  verify_rows streams the [B*N, V] logits (the only large
// input) once, in chunks of kVChunk tokens per CTA, and leaves per chunk the
// max logit, its lowest index and, for typical acceptance, the partial sums
// sum exp(z/T - m) and sum exp(z/T - m) * z/T.  verify_path, one CTA per
// sequence, merges the chunks per node and runs the integer path selection.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <type_traits>

#include "abi_internal.h"
#include "common.cuh"
#include "kv_compact.cuh"

namespace medusa {

constexpr int kVChunk = 4096;   // tokens per warp work item
constexpr int kRowWarps = 8;    // work items per CTA

template <typename T>
struct Elt;
template <>
struct Elt<__nv_bfloat16> {
  static constexpr int kPerVec = 8;  // elements per 16-byte load
  static constexpr uint32_t kNegInf = 0xFF80u;
  __device__ static float get(const uint4& r, int e) {
    const uint32_t w = (&r.x)[e >> 1];
    return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
  }
  __device__ static uint4 load_scalar(const __nv_bfloat16* p, int n) {
    uint16_t h[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) h[e] = e < n ? reinterpret_cast<const uint16_t*>(p)[e] : 0xFF80u;
    uint4 r;
    r.x = h[0] | (uint32_t(h[1]) << 16);
    r.y = h[2] | (uint32_t(h[3]) << 16);
    r.z = h[4] | (uint32_t(h[5]) << 16);
    r.w = h[6] | (uint32_t(h[7]) << 16);
    return r;
  }
};
template <>
struct Elt<float> {
  static constexpr int kPerVec = 4;
  __device__ static float get(const uint4& r, int e) { return __uint_as_float((&r.x)[e]); }
  __device__ static uint4 load_scalar(const float* p, int n) {
    uint4 r;
    uint32_t* w = &r.x;
#pragma unroll
    for (int e = 0; e < 4; ++e) w[e] = e < n ? __float_as_uint(p[e]) : 0xFF800000u;
    return r;
  }
};

// paired fp32 arithmetic (two lanes in one 64-bit register, sm_100) and the
// SFU's 2^x (relative error about 2^-22; -inf -> 0)
__device__ __forceinline__ uint64_t f32x2_pack_v(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f32x2_unpack_v(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f32x2_fma_v(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_add_v(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float ex2_approx_v(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <typename T>
__device__ __forceinline__ float load1(const T* p);
template <>
__device__ __forceinline__ float load1<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <>
__device__ __forceinline__ float load1<float>(const float* p) {
  return *p;
}

// One warp per (row, 4096-token chunk) work item: every lane issues all its
// 16-byte loads at once, then the warp reduces with shuffles only.
template <typename T, bool TYPICAL>
__device__ __forceinline__ void verify_item(const T* __restrict__ logits, int V, int n_chunks,
                                            long long item, int lane, float inv_T,
                                            RowPart* __restrict__ part, int32_t* status) {
  using E = Elt<T>;
  constexpr int EV = E::kPerVec;
  constexpr int NL = kVChunk / (32 * EV);  // loads per lane
  const long long row = item / n_chunks;
  const int c = static_cast<int>(item - row * n_chunks);
  const T* base = logits + row * V;
  const int v0 = c * kVChunk;
  const bool vec = (V % EV) == 0;
  uint4 raw[NL];
#pragma unroll
  for (int r = 0; r < NL; ++r) {
    const int e0 = v0 + (r * 32 + lane) * EV;
    if (vec && e0 + EV <= V) {
      raw[r] = ld_stream16(base + e0);
    } else {
      raw[r] = E::load_scalar(base + e0, e0 < V ? min(EV, V - e0) : 0);
    }
  }
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    // bf16: packed maximum (NaN propagates, so one check at the end catches a
    // NaN anywhere), then the first index holding that value
    __nv_bfloat162 m2 = __halves2bfloat162(__ushort_as_bfloat16(0xFF80u), __ushort_as_bfloat16(0xFF80u));
#pragma unroll
    for (int r = 0; r < NL; ++r) {
      const __nv_bfloat162* w = reinterpret_cast<const __nv_bfloat162*>(&raw[r].x);
      m2 = __hmax2_nan(m2, __hmax2_nan(__hmax2_nan(w[0], w[1]), __hmax2_nan(w[2], w[3])));
    }
    const float lo_f = __low2float(m2), hi_f = __high2float(m2);
    bool nan = (lo_f != lo_f) || (hi_f != hi_f);
    float M = fmaxf(lo_f, hi_f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (__any_sync(0xffffffffu, nan)) {
      if (lane == 0) report(status, MEDUSA_ERR_DEVICE_CHECK);
    }
    // first index holding M: a floating equality (so +0 and -0 both match
    // a zero maximum) on each load's packed maximum (recomputed: keeping
    // them would cost registers and so loads in flight), then inside the
    // first load that holds M
    const __nv_bfloat162 M2 = __float2bfloat162_rn(M);  // exact: M is a bf16 value
    int idx = 0x7fffffff;
#pragma unroll
    for (int r = NL - 1; r >= 0; --r) {
      const __nv_bfloat162* w = reinterpret_cast<const __nv_bfloat162*>(&raw[r].x);
      const __nv_bfloat162 e =
          __heq2(__hmax2(__hmax2(w[0], w[1]), __hmax2(w[2], w[3])), M2);
      if (*reinterpret_cast<const uint32_t*>(&e) != 0u) {  // rare: the load holding M
        int k = 8;
#pragma unroll
        for (int q = 3; q >= 0; --q) {
          const __nv_bfloat162 eq = __heq2(w[q], M2);
          const uint32_t eb = *reinterpret_cast<const uint32_t*>(&eq);
          if (eb & 0xFFFF0000u) k = 2 * q + 1;
          if (eb & 0x0000FFFFu) k = 2 * q;
        }
        idx = v0 + (r * 32 + lane) * EV + k;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) idx = min(idx, __shfl_xor_sync(0xffffffffu, idx, o));
    float ss = 0.f, tt = 0.f;
    if constexpr (TYPICAL) {
      // typical: s = sum exp(z/T - M/T) and t = sum exp(z/T - M/T) * z/T, as
      // 2^(z * log2(e)/T - M * log2(e)/T) on paired fp32 instructions and the
      // SFU; padding (-inf) contributes 0 to both
      const float cl = inv_T * 1.4426950408889634f;
      const uint64_t c2 = f32x2_pack_v(cl, cl);
      const uint64_t nb2 = f32x2_pack_v(-M * cl, -M * cl);
      const uint64_t it2 = f32x2_pack_v(inv_T, inv_T);
      uint64_t s2[2] = {0ull, 0ull}, t2[2] = {0ull, 0ull};
#pragma unroll
      for (int r = 0; r < NL; ++r) {
        const uint32_t* w = &raw[r].x;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float z0 = __uint_as_float(w[q] << 16), z1 = __uint_as_float(w[q] & 0xffff0000u);
          const uint64_t z2 = f32x2_pack_v(z0, z1);
          float x0, x1;
          f32x2_unpack_v(f32x2_fma_v(z2, c2, nb2), x0, x1);
          const float e0 = ex2_approx_v(x0), e1 = ex2_approx_v(x1);
          float zt0, zt1;
          f32x2_unpack_v(f32x2_fma_v(z2, it2, 0ull), zt0, zt1);
          zt0 = z0 == -INFINITY ? 0.f : zt0;
          zt1 = z1 == -INFINITY ? 0.f : zt1;
          const uint64_t e2 = f32x2_pack_v(e0, e1);
          s2[q & 1] = f32x2_add_v(s2[q & 1], e2);
          t2[q & 1] = f32x2_fma_v(e2, f32x2_pack_v(zt0, zt1), t2[q & 1]);
        }
      }
      float a0, a1, b0, b1;
      f32x2_unpack_v(f32x2_add_v(s2[0], s2[1]), a0, a1);
      f32x2_unpack_v(f32x2_add_v(t2[0], t2[1]), b0, b1);
      ss = a0 + a1;
      tt = b0 + b1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        tt += __shfl_xor_sync(0xffffffffu, tt, o);
      }
    }
    if (lane == 0) {
      RowPart rp;
      rp.maxz = M;
      rp.idx = idx;
      rp.s = ss;
      rp.t = tt;
      part[row * n_chunks + c] = rp;
    }
    return;
  }
  // best (largest, lowest index) of this lane: indices ascend in (r, e) order
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  bool nan = false;
#pragma unroll
  for (int r = 0; r < NL; ++r) {
    const int e0 = v0 + (r * 32 + lane) * EV;
#pragma unroll
    for (int e = 0; e < EV; ++e) {
      const float x = E::get(raw[r], e);
      nan |= (x != x);
      if (e0 + e < V && better(x, e0 + e, bv, bi)) {
        bv = x;
        bi = e0 + e;
      }
    }
  }
  if (nan) report(status, MEDUSA_ERR_DEVICE_CHECK);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (better(ov, oi, bv, bi)) {
      bv = ov;
      bi = oi;
    }
  }
  float ss = 0.f, tt = 0.f;
  if (TYPICAL) {
    const float m = bv * inv_T;
#pragma unroll
    for (int r = 0; r < NL; ++r) {
#pragma unroll
      for (int e = 0; e < EV; ++e) {
        const float x = E::get(raw[r], e);
        if (x != -INFINITY) {
          const float zt = x * inv_T;
          const float w = expf(zt - m);
          ss += w;
          tt += w * zt;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      tt += __shfl_xor_sync(0xffffffffu, tt, o);
    }
  }
  if (lane == 0) {
    RowPart rp;
    rp.maxz = bv;
    rp.idx = bi;
    rp.s = ss;
    rp.t = tt;
    part[row * n_chunks + c] = rp;
  }
}

// Persistent grid (a few CTAs per SM): each warp takes items warp, warp +
// total warps, ... so that no partial last wave of CTAs is left.
template <typename T, bool TYPICAL>
__global__ void __launch_bounds__(kRowWarps * 32,
                                  std::is_same<T, __nv_bfloat16>::value ? 3 : 1)
    verify_rows_kernel(const T* __restrict__ logits, int V, int n_chunks, long long n_items,
                       float inv_T, RowPart* __restrict__ part, int32_t* status) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  for (long long item = (long long)blockIdx.x * kRowWarps + (threadIdx.x >> 5); item < n_items;
       item += (long long)gridDim.x * kRowWarps)
    verify_item<T, TYPICAL>(logits, V, n_chunks, item, lane, inv_T, part, status);
}

// One CTA of kPathThreads per sequence.  The chunk records of node i are
// merged by a group of tpn consecutive threads (tpn a power of two, tpn * N <=
// kPathThreads), each taking every tpn-th chunk, then shuffles within the
// group; the path logic runs on threads 0..N-1.
constexpr int kPathThreads = 1024;

template <typename T>
__global__ void __launch_bounds__(kPathThreads)
    verify_path_kernel(const T* __restrict__ logits, const __nv_bfloat16* __restrict__ hidden,
                       const __nv_bfloat16* __restrict__ lm_head, int d,
                       const RowPart* __restrict__ part, int n_chunks, long long row_stride,
                       long long chunk_stride, int tpn, const float* __restrict__ cand_logit,
                       const int32_t* __restrict__ cand_ids,
                       const int32_t* __restrict__ parent, const int32_t* __restrict__ depth,
                       int N, int max_depth, int V, int typical, float inv_T, float eps,
                       float delta, int32_t* __restrict__ accept_len,
                       int32_t* __restrict__ accepted_nodes, int32_t* __restrict__ accepted_tokens,
                       int32_t* __restrict__ bonus, int32_t* status, CompactArgs ca) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ int s_g[MEDUSA_MAX_NODES];
  __shared__ float s_lse[MEDUSA_MAX_NODES];
  __shared__ float s_logthr[MEDUSA_MAX_NODES];
  __shared__ int s_parent[MEDUSA_MAX_NODES];
  __shared__ int s_depth[MEDUSA_MAX_NODES];
  __shared__ int s_pass[MEDUSA_MAX_NODES];
  __shared__ float s_zc[MEDUSA_MAX_NODES];  // logit of node i's candidate at its parent
  __shared__ int s_cand[MEDUSA_MAX_NODES];
  __shared__ int s_best;
  __shared__ int s_bad;
  __shared__ int s_src[MEDUSA_MAX_HEADS + 1];  // kept branch's cache slots (compaction)
  __shared__ int s_keep, s_prefix;
  const int b = blockIdx.x;
  const int i = threadIdx.x;
  if (i == 0) {
    s_best = 0xFFFF;  // the root: depth 0, node 0
    s_bad = 0;
  }
  // the tree, the candidates and the chunk records are read in one round trip
  if (i < N) {
    s_parent[i] = parent[i];
    s_depth[i] = depth[i];
    s_cand[i] = cand_ids[(size_t)b * N + i];
  }
  {
    // merge the chunks of row (b, node): this thread's share, then the group
    const int node = i / tpn, sub = i - node * tpn;
    const bool active = node < N;
    const RowPart* rp = part + ((size_t)b * N + (active ? node : 0)) * row_stride;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    float Mt = -INFINITY, S = 0.f, Tt = 0.f;  // sums relative to exp(Mt)
    if (active) {
      for (int c = sub; c < n_chunks; c += tpn) {
        const RowPart q = rp[c * chunk_stride];
        if (better(q.maxz, q.idx, bv, bi)) {
          bv = q.maxz;
          bi = q.idx;
        }
        if (typical) {
          const float mq = q.maxz * inv_T;
          if (mq > Mt) {
            const float w = Mt == -INFINITY ? 0.f : expf(Mt - mq);
            S = S * w + q.s;
            Tt = Tt * w + q.t;
            Mt = mq;
          } else if (mq != -INFINITY) {
            const float w = expf(mq - Mt);
            S += q.s * w;
            Tt += q.t * w;
          }
        }
      }
    }
    for (int o = 1; o < tpn; o <<= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
      if (typical) {
        const float oM = __shfl_xor_sync(0xffffffffu, Mt, o);
        const float oS = __shfl_xor_sync(0xffffffffu, S, o);
        const float oT = __shfl_xor_sync(0xffffffffu, Tt, o);
        const float nM = fmaxf(Mt, oM);
        const float wa = Mt == -INFINITY ? 0.f : expf(Mt - nM);
        const float wb = oM == -INFINITY ? 0.f : expf(oM - nM);
        S = S * wa + oS * wb;
        Tt = Tt * wa + oT * wb;
        Mt = nM;
      }
    }
    if (active && sub == 0) {
      s_g[node] = bi;
      if (typical) {
        const float lse = Mt + logf(S);
        const float H = lse - Tt / S;
        const float thr = fminf(eps, delta * expf(-H));
        s_lse[node] = lse;
        s_logthr[node] = thr > 0.f ? logf(thr) : -INFINITY;
      }
    }
  }
  __syncthreads();
  if (i < N) {
    const int pa = s_parent[i];
    const int dp = s_depth[i];
    const bool ok = (i == 0) ? (pa == -1 && dp == 0)
                             : (pa >= 0 && pa < i && dp == s_depth[pa] + 1 && dp <= max_depth);
    if (!ok) atomicOr(&s_bad, 1);
  }
  __syncthreads();
  if (s_bad) {
    if (i == 0) {
      report(status, MEDUSA_ERR_DEVICE_CHECK);
      accept_len[b] = 0;
    }
    return;
  }
  if (typical && logits == nullptr && cand_logit == nullptr) {
    // no materialised logits: z = lm_head[tok] . hidden[b, parent], one warp
    // per node, 16-byte loads (d is a multiple of 64)
    const int warp = i >> 5, lane = i & 31;
    for (int c = 1 + warp; c < N; c += kPathThreads / 32) {
      const int tok = s_cand[c];
      float acc = 0.f;
      if (tok >= 0 && tok < V) {
        const uint4* wr = reinterpret_cast<const uint4*>(lm_head + (size_t)tok * d);
        const uint4* hr =
            reinterpret_cast<const uint4*>(hidden + ((size_t)b * N + s_parent[c]) * d);
        for (int e = lane; e < d / 8; e += 32) {
          const uint4 x = wr[e], y = hr[e];
          const uint32_t* xw = &x.x;
          const uint32_t* yw = &y.x;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[q]));
            const float2 yf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&yw[q]));
            acc = fmaf(xf.x, yf.x, acc);
            acc = fmaf(xf.y, yf.y, acc);
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) s_zc[c] = acc;
    }
    __syncthreads();
  }
  if (i < N) {
    int pass = 1;
    if (i > 0) {
      const int tok = s_cand[i];
      const int pa = s_parent[i];
      if (tok < 0 || tok >= V) {
        report(status, MEDUSA_ERR_DEVICE_CHECK);
        pass = 0;
      } else if (!typical) {
        pass = s_g[pa] == tok;
      } else {
        const float z = logits != nullptr       ? load1<T>(logits + ((size_t)b * N + pa) * V + tok)
                        : cand_logit != nullptr ? cand_logit[(size_t)b * N + i]
                                                : s_zc[i];
        const float lp = z * inv_T - s_lse[pa];
        pass = lp > s_logthr[pa];
      }
    }
    s_pass[i] = pass;
  }
  __syncthreads();
  if (i < N) {
    bool acc = true;
    for (int j = i; j > 0 && acc; j = s_parent[j]) acc = s_pass[j] != 0;
    if (acc) atomicMax(&s_best, (s_depth[i] << 16) | (0xFFFF - i));
  }
  __syncthreads();
  if (i == 0) {
    const int best = 0xFFFF - (s_best & 0xFFFF);
    const int L = s_depth[best];
    const size_t o = (size_t)b * (max_depth + 1);
    for (int t = L + 1; t <= max_depth; ++t) {
      accepted_nodes[o + t] = -1;
      accepted_tokens[o + t] = -1;
    }
    for (int j = best; j >= 0; j = s_parent[j]) {
      accepted_nodes[o + s_depth[j]] = j;
      if (j > 0) accepted_tokens[o + s_depth[j] - 1] = s_cand[j];
    }
    accepted_tokens[o + L] = s_g[best];
    accept_len[b] = L;
    bonus[b] = s_g[best];
    if (ca.Kc != nullptr) {
      // the kept branch's cache slots, for the compaction below
      const int P = ca.prefix_len[b];
      bool ok = P >= 0;
      for (int j = best; j >= 0; j = s_parent[j]) {
        const long long slot = (long long)P + j;
        if (slot >= ca.cap) ok = false;
        s_src[s_depth[j]] = (int)slot;
      }
      s_keep = ok ? L : -1;
      s_prefix = P;
      if (!ok) report(status, MEDUSA_ERR_DEVICE_CHECK);
    }
  }
  if (ca.Kc == nullptr) return;
  // Compaction of the kept branch by the same block (one launch less than a
  // separate compaction call): for j = 0..L, slot P + j <- slot P + node_j.
  __syncwarp();  // warp 0 reconverges: its lane 0 ran the path alone
  __syncthreads();
  if (s_keep < 0) return;
  extern __shared__ __align__(16) uint4 stage[];
  compact_sequence(ca, b, s_prefix, s_keep, s_src, max_depth + 1, stage);
}

// CTAs for the persistent row kernel: as many as stay resident, fewer when
// there are fewer work items
template <typename K>
static unsigned rows_grid(K kernel, long long n_items) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kRowWarps * 32, 0) !=
          cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  const long long resident = (long long)per_sm * device_sm_count();
  const long long need = (n_items + kRowWarps - 1) / kRowWarps;
  return (unsigned)(need < resident ? need : resident);
}

int path_threads_per_node(int N, int n_chunks) {
  int tpn = 1;  // threads merging one node's chunks
  while (tpn < 32 && tpn * 2 * N <= kPathThreads && tpn < n_chunks) tpn *= 2;
  return tpn;
}

medusa_status_t verify_path_from_parts(const RowPart* part, int n_chunks,
                                       const __nv_bfloat16* hidden,
                                       const __nv_bfloat16* lm_head, int d,
                                       const int32_t* cand_ids, const medusa_tree_t& tree, int B,
                                       int V, medusa_accept_t mode, float temperature, float eps,
                                       float delta, int32_t* accept_len,
                                       int32_t* accepted_nodes, int32_t* accepted_tokens,
                                       int32_t* bonus, int32_t* status, cudaStream_t stream) {
  const int N = tree.n_nodes;
  const bool typical = mode == MEDUSA_ACCEPT_TYPICAL;
  const float inv_T = typical ? 1.0f / temperature : 1.0f;
  launch(verify_path_kernel<__nv_bfloat16>, B, kPathThreads, 0, stream, nullptr, hidden, lm_head, d,
         part, n_chunks, n_chunks, 1, path_threads_per_node(N, n_chunks), nullptr, cand_ids,
         tree.parent, tree.depth, N, tree.max_depth, V, typical ? 1 : 0, inv_T, eps, delta,
         accept_len, accepted_nodes, accepted_tokens, bonus, status, CompactArgs{});
  return check_launch("verify_path");
}

// One record per row from a vocabulary shard's chunk records (merged in
// chunk order, like the path kernel's merge), token ids moved to global by
// v_offset; and each node's candidate logit at its parent when the candidate
// token lies in this shard (-inf otherwise, and for the root).
template <typename T>
__global__ void __launch_bounds__(256)
    shard_records_kernel(const T* __restrict__ logits, const RowPart* __restrict__ part,
                         int n_chunks, const int32_t* __restrict__ cand_ids,
                         const int32_t* __restrict__ parent, int B, int N, int V_shard,
                         int v_offset, int typical, float inv_T, RowPart* __restrict__ records,
                         float* __restrict__ cand_logit, int32_t* status) {
  grid_dep_wait();
  grid_dep_launch();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= B * N) return;
  const RowPart* rp = part + (size_t)r * n_chunks;
  RowPart o;
  o.maxz = -INFINITY;
  o.idx = 0x7fffffff;
  o.s = 0.f;
  o.t = 0.f;
  float Mt = -INFINITY;
  for (int c = 0; c < n_chunks; ++c) {
    const RowPart q = rp[c];
    if (better(q.maxz, q.idx, o.maxz, o.idx)) {
      o.maxz = q.maxz;
      o.idx = q.idx;
    }
    if (typical) {
      const float mq = q.maxz * inv_T;
      if (mq > Mt) {
        const float w = Mt == -INFINITY ? 0.f : expf(Mt - mq);
        o.s = o.s * w + q.s;
        o.t = o.t * w + q.t;
        Mt = mq;
      } else if (mq != -INFINITY) {
        const float w = expf(mq - Mt);
        o.s += q.s * w;
        o.t += q.t * w;
      }
    }
  }
  if (o.idx != 0x7fffffff) o.idx += v_offset;
  records[r] = o;
  const int b = r / N, i = r - b * N;
  float z = -INFINITY;
  if (i > 0) {
    const int pa = parent[i];
    const int tok = cand_ids[r];
    if (pa < 0 || pa >= N) {
      report(status, MEDUSA_ERR_DEVICE_CHECK);
    } else if (tok >= v_offset && tok < v_offset + V_shard) {
      z = load1<T>(logits + ((size_t)b * N + pa) * V_shard + (tok - v_offset));
    }
  }
  cand_logit[r] = z;
}

size_t verify_records_workspace_size(int B, int N, int V_shard) {
  return verify_accept_workspace_size(B, N, V_shard);
}

medusa_status_t verify_records(const void* logits, medusa_dtype_t dt, const int32_t* cand_ids,
                               const medusa_tree_t& tree, int B, int V_shard, int v_offset,
                               medusa_accept_t mode, float temperature, RowPart* records,
                               float* cand_logit, void* ws, int32_t* status, cudaStream_t stream) {
  const int N = tree.n_nodes;
  const int n_chunks = (V_shard + kVChunk - 1) / kVChunk;
  RowPart* part = static_cast<RowPart*>(ws);
  const bool typical = mode == MEDUSA_ACCEPT_TYPICAL;
  const float inv_T = typical ? 1.0f / temperature : 1.0f;
  const long long n_items = (long long)B * N * n_chunks;
  const int grid = (B * N + 255) / 256;
  if (dt == MEDUSA_BF16) {
    const __nv_bfloat16* lg = static_cast<const __nv_bfloat16*>(logits);
    if (typical) {
      auto k = verify_rows_kernel<__nv_bfloat16, true>;
      launch(k, rows_grid(k, n_items), kRowWarps * 32, 0, stream, lg, V_shard, n_chunks, n_items,
             inv_T, part, status);
    } else {
      auto k = verify_rows_kernel<__nv_bfloat16, false>;
      launch(k, rows_grid(k, n_items), kRowWarps * 32, 0, stream, lg, V_shard, n_chunks, n_items,
             inv_T, part, status);
    }
    launch(shard_records_kernel<__nv_bfloat16>, grid, 256, 0, stream, lg, part, n_chunks, cand_ids,
           tree.parent, B, N, V_shard, v_offset, typical ? 1 : 0, inv_T, records, cand_logit,
           status);
  } else {
    const float* lg = static_cast<const float*>(logits);
    if (typical) {
      auto k = verify_rows_kernel<float, true>;
      launch(k, rows_grid(k, n_items), kRowWarps * 32, 0, stream, lg, V_shard, n_chunks, n_items,
             inv_T, part, status);
    } else {
      auto k = verify_rows_kernel<float, false>;
      launch(k, rows_grid(k, n_items), kRowWarps * 32, 0, stream, lg, V_shard, n_chunks, n_items,
             inv_T, part, status);
    }
    launch(shard_records_kernel<float>, grid, 256, 0, stream, lg, part, n_chunks, cand_ids,
           tree.parent, B, N, V_shard, v_offset, typical ? 1 : 0, inv_T, records, cand_logit,
           status);
  }
  return check_launch("verify_records");
}

medusa_status_t verify_from_records(const RowPart* records, int G, const float* cand_logit,
                                    const int32_t* cand_ids, const medusa_tree_t& tree, int B,
                                    int V, medusa_accept_t mode, float temperature, float eps,
                                    float delta, int32_t* accept_len, int32_t* accepted_nodes,
                                    int32_t* accepted_tokens, int32_t* bonus, int32_t* status,
                                    cudaStream_t stream) {
  const int N = tree.n_nodes;
  const bool typical = mode == MEDUSA_ACCEPT_TYPICAL;
  const float inv_T = typical ? 1.0f / temperature : 1.0f;
  // records are shard-major: [G][B * N]
  launch(verify_path_kernel<float>, B, kPathThreads, 0, stream, nullptr, nullptr, nullptr, 0,
         records, G, 1, (long long)B * N, path_threads_per_node(N, G), cand_logit, cand_ids,
         tree.parent, tree.depth, N, tree.max_depth, V, typical ? 1 : 0, inv_T, eps, delta,
         accept_len, accepted_nodes, accepted_tokens, bonus, status, CompactArgs{});
  return check_launch("verify_path");
}

size_t verify_accept_workspace_size(int B, int N, int V) {
  const size_t n_chunks = (size_t)(V + kVChunk - 1) / kVChunk;
  return align256((size_t)B * N * n_chunks * sizeof(RowPart));
}

medusa_status_t verify_accept(const void* logits, medusa_dtype_t dt, const int32_t* cand_ids,
                              const medusa_tree_t& tree, int B, int V, medusa_accept_t mode,
                              float temperature, float eps, float delta, int32_t* accept_len,
                              int32_t* accepted_nodes, int32_t* accepted_tokens, int32_t* bonus,
                              void* ws, int32_t* status, cudaStream_t stream,
                              const CompactArgs& ca, size_t ca_smem) {
  const int N = tree.n_nodes;
  // the compaction tail's staging memory
  if (ca_smem > 48 * 1024) {
    const cudaError_t e =
        dt == MEDUSA_BF16
            ? cudaFuncSetAttribute(verify_path_kernel<__nv_bfloat16>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ca_smem)
            : cudaFuncSetAttribute(verify_path_kernel<float>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ca_smem);
    if (e != cudaSuccess) return fail(MEDUSA_ERR_CUDA, "cudaFuncSetAttribute(verify_path) failed");
  }
  const int n_chunks = (V + kVChunk - 1) / kVChunk;
  RowPart* part = static_cast<RowPart*>(ws);
  const bool typical = mode == MEDUSA_ACCEPT_TYPICAL;
  const float inv_T = typical ? 1.0f / temperature : 1.0f;
  const long long n_items = (long long)B * N * n_chunks;
  const int tpn = path_threads_per_node(N, n_chunks);
  if (dt == MEDUSA_BF16) {
    const __nv_bfloat16* lg = static_cast<const __nv_bfloat16*>(logits);
    if (typical) {
      auto k = verify_rows_kernel<__nv_bfloat16, true>;
      launch(k, rows_grid(k, n_items), kRowWarps * 32, 0, stream, lg, V, n_chunks, n_items, inv_T,
             part, status);
    } else {
      auto k = verify_rows_kernel<__nv_bfloat16, false>;
      launch(k, rows_grid(k, n_items), kRowWarps * 32, 0, stream, lg, V, n_chunks, n_items, inv_T,
             part, status);
    }
    medusa_status_t st = check_launch("verify_rows");
    if (st != MEDUSA_OK) return st;
    launch(verify_path_kernel<__nv_bfloat16>, B, kPathThreads, ca_smem, stream, lg, nullptr, nullptr,
           0, part, n_chunks, n_chunks, 1, tpn, nullptr, cand_ids, tree.parent, tree.depth, N,
           tree.max_depth, V, typical ? 1 : 0, inv_T, eps, delta, accept_len, accepted_nodes,
           accepted_tokens, bonus, status, ca);
    return check_launch("verify_path");
  }
  const float* lg = static_cast<const float*>(logits);
  if (typical) {
    auto k = verify_rows_kernel<float, true>;
    launch(k, rows_grid(k, n_items), kRowWarps * 32, 0, stream, lg, V, n_chunks, n_items, inv_T,
           part, status);
  } else {
    auto k = verify_rows_kernel<float, false>;
    launch(k, rows_grid(k, n_items), kRowWarps * 32, 0, stream, lg, V, n_chunks, n_items, inv_T,
           part, status);
  }
  medusa_status_t st = check_launch("verify_rows");
  if (st != MEDUSA_OK) return st;
  launch(verify_path_kernel<float>, B, kPathThreads, ca_smem, stream, lg, nullptr, nullptr, 0, part,
         n_chunks, n_chunks, 1, tpn, nullptr, cand_ids, tree.parent, tree.depth, N, tree.max_depth,
         V, typical ? 1 : 0, inv_T, eps, delta, accept_len, accepted_nodes, accepted_tokens, bonus,
         status, ca);
  return check_launch("verify_path");
}

}  // namespace medusa

// ---------------------------------------------------------------------------
// medusa_verify_accept_noalloc: the same verification with no caller-supplied
// workspace.  Some callers cannot hand this library device memory per call:
// a host framework that owns and pre-reserves all device memory and forbids
// growing it at run time, or code that must not call cudaMalloc/cudaFree on
// the hot path because those calls can synchronise the device.  For them the
// per-chunk row statistics live in a fixed array compiled into the library.
// ---------------------------------------------------------------------------
namespace {

// 4 MiB holds B * N * ceil(V / 4096) 16-byte row records up to 262144 records
// (for example B = 32, N = 128, V = 128256 needs 131072).  Every GPU that loads the library
// keeps this array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_verify_noalloc_scratch[kNoAllocScratchBytes];

}  // namespace

extern "C" medusa_status_t medusa_verify_accept_noalloc(
    const void* logits, medusa_dtype_t dt, const int32_t* cand_ids, const medusa_tree_t* tree,
    int B, int V, medusa_accept_t mode, float temperature, float eps, float delta,
    int32_t* accept_len, int32_t* accepted_nodes, int32_t* accepted_tokens, int32_t* bonus,
    int32_t* dev_status, void* stream) {
  // the checks of medusa_verify_accept first, so that a bad tree or shape
  // gets the same error here as there; then the scratch limit
  medusa_status_t st = medusa::check_verify_accept_args(logits, dt, cand_ids, tree, B, V, mode,
                                                        temperature, eps, delta, accept_len,
                                                        accepted_nodes, accepted_tokens, bonus);
  if (st != MEDUSA_OK) return st;
  if (medusa::verify_accept_workspace_size(B, tree->n_nodes, V) > kNoAllocScratchBytes)
    return medusa::fail(MEDUSA_ERR_WORKSPACE,
                        "verify_accept_noalloc: B * n_nodes * ceil(V / 4096) * 16 bytes exceeds "
                        "the 4 MiB static scratch; use medusa_verify_accept with a workspace");
  // Host code sees only a stand-in for the device array.  Its device address
  // is looked up on every call, with the caller's device and context current:
  // the lookup is a host-side query (no synchronisation), and an address kept
  // from an earlier call could belong to a module that a device reset or
  // another context has since replaced.
  void* scratch = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&scratch, g_verify_noalloc_scratch);
  if (e != cudaSuccess || scratch == nullptr) {
    cudaGetLastError();
    return medusa::fail(MEDUSA_ERR_CUDA,
                        "verify_accept_noalloc: cudaGetSymbolAddress of the scratch failed");
  }
  // every row record is written by the row kernel before the path kernel
  // reads it, so the scratch needs no clearing between calls
  return medusa_verify_accept(logits, dt, cand_ids, tree, B, V, mode, temperature, eps, delta,
                              accept_len, accepted_nodes, accepted_tokens, bonus, scratch,
                              kNoAllocScratchBytes, dev_status, stream);
}
