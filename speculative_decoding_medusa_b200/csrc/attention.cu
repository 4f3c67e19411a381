// Tree attention: every tree node attends to the cached prefix and to its
// own ancestors (and itself) in the tree.
//
// "Medusa Heads" glossary, "Attention arborescente et acceptation": all
// candidate tokens are appended to the input at once; a mask lets each one see
// only its ancestors, so one forward pass scores every branch.
//
// bf16 path: split-KV.  For each (sequence b, kv head) the N*G query rows
// (G = Hq/Hkv grouped query heads per kv head) form tiles of 64 rows; the
// prefix is cut into chunks of `chunk` keys, plus one more split for the N
// tree keys (read from k_new/v_new, masked by the ancestor bitmask).  Each CTA
// keeps an online softmax and writes a normalised partial output and its
// log2-sum-exp; a combine kernel merges the splits.  The tree split with query
// tile 0 also writes the tree K/V into cache slots P + i.
// QK^T and PV run on mma.sync m16n8k16 (bf16, fp32 accumulate); the softmax
// weights enter PV as two bf16 terms (hi + lo) to keep ~16 mantissa bits.
//
// fp32 path: one warp per query row on CUDA cores (small shapes).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "abi_internal.h"
#include "common.cuh"

namespace medusa {

constexpr int kBM = 64;  // query rows per CTA (4 warps x 16)
constexpr int kBN = 64;  // keys per tile
constexpr int kAttnThreads = 128;

struct AttnParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* Kc;
  __nv_bfloat16* Vc;
  const int32_t* prefix_len;
  const uint32_t* anc_mask;
  float* o_part;   // [B*Hkv, n_qt, S, kBM, DH]
  float* lse_part; // [B*Hkv, n_qt, S, kBM]
  int B, N, Hq, Hkv, G, R, n_qt, S, chunk, cap, max_prefix, words;
  float scale_log2;
  int32_t* status;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// split x into bf16 hi + bf16 lo (x ~= hi + lo)
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float r0 = x0 - __low2float(h);
  const float r1 = x1 - __high2float(h);
  hi = *reinterpret_cast<uint32_t*>(&h);
  lo = pack_bf16(r0, r1);
}

// byte offset of 16-byte chunk `c` of row `r` in a [rows][DH] bf16 tile whose
// chunks are XOR-swizzled by the row (conflict-free ldmatrix)
template <int DH>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * (DH * 2) + ((c ^ (r & 7)) << 4));
}

template <int DH>
__global__ void __launch_bounds__(kAttnThreads, 2) tree_attn_bf16_kernel(AttnParams p) {
  constexpr int CH = DH / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kBM * DH * 2;
  uint8_t* sV = sK + 2 * kBN * DH * 2;
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sV + 2 * kBN * DH * 2);  // [kBM][8]

  const int s = blockIdx.x;
  const int qt = blockIdx.y;
  const int bh = blockIdx.z;
  const int b = bh / p.Hkv;
  const int kvh = bh - b * p.Hkv;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const int P = p.prefix_len[b];
  if (P < 0 || P > p.max_prefix || P + p.N > p.cap) {
    if (tid == 0) report(p.status, MEDUSA_ERR_DEVICE_CHECK);
    return;
  }
  const int n_pre = (P + p.chunk - 1) / p.chunk;
  if (s > n_pre) return;
  const bool tree_split = (s == n_pre);
  const int key0 = tree_split ? 0 : s * p.chunk;
  const int key_end = tree_split ? p.N : min(P, key0 + p.chunk);
  const int n_tiles = (key_end - key0 + kBN - 1) / kBN;

  const size_t kv_head_base = ((size_t)b * p.Hkv + kvh) * p.cap;  // in rows of DH
  // ---- tree split, tile 0: write the tree K/V into the cache ----
  if (tree_split && qt == 0) {
    for (int e = tid; e < p.N * CH; e += kAttnThreads) {
      const int j = e / CH, c = e - j * CH;
      const size_t src = (((size_t)b * p.N + j) * p.Hkv + kvh) * DH + c * 8;
      const size_t dst = (kv_head_base + P + j) * DH + c * 8;
      *reinterpret_cast<uint4*>(p.Kc + dst) = *reinterpret_cast<const uint4*>(p.k_new + src);
      *reinterpret_cast<uint4*>(p.Vc + dst) = *reinterpret_cast<const uint4*>(p.v_new + src);
    }
  }

  // ---- Q tile (rows r = qt*kBM + row; node r / G, head kvh*G + r % G) ----
  const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
  for (int e = tid; e < kBM * CH; e += kAttnThreads) {
    const int row = e / CH, c = e - row * CH;
    const int r = qt * kBM + row;
    const bool valid = r < p.R;
    const int node = valid ? r / p.G : 0;
    const int g = valid ? r - node * p.G : 0;
    const __nv_bfloat16* src = p.q + (((size_t)b * p.N + node) * p.Hq + kvh * p.G + g) * DH + c * 8;
    cp_async16(sQa + swz<DH>(row, c), valid ? src : p.q, valid);
  }
  if (tree_split) {
    for (int e = tid; e < kBM * 8; e += kAttnThreads) {
      const int row = e >> 3, w = e & 7;
      const int r = qt * kBM + row;
      uint32_t m = 0xffffffffu;
      if (r < p.R && w < p.words) m = p.anc_mask[(size_t)(r / p.G) * p.words + w];
      sMask[e] = m;
    }
  }

  auto load_tile = [&](int t, int stage) {
    const int k0 = key0 + t * kBN;
    for (int e = tid; e < kBN * CH; e += kAttnThreads) {
      const int row = e / CH, c = e - row * CH;
      const int key = k0 + row;
      const bool valid = key < key_end;
      const __nv_bfloat16 *ks, *vs;
      if (tree_split) {
        const size_t off = (((size_t)b * p.N + key) * p.Hkv + kvh) * DH + c * 8;
        ks = valid ? p.k_new + off : p.k_new;
        vs = valid ? p.v_new + off : p.v_new;
      } else {
        const size_t off = (kv_head_base + key) * DH + c * 8;
        ks = valid ? p.Kc + off : p.Kc;
        vs = valid ? p.Vc + off : p.Vc;
      }
      const uint32_t so = stage * kBN * DH * 2 + swz<DH>(row, c);
      cp_async16(sKa + so, ks, valid);
      cp_async16(sVa + so, vs, valid);
    }
  };

  load_tile(0, 0);
  cp_async_commit();  // group 0: Q + tile 0

  // per-thread state: rows r_lo = 16*warp + lane/4 and r_hi = r_lo + 8
  float o[DH / 8][4];
#pragma unroll
  for (int n = 0; n < DH / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
  uint32_t qf[DH / 16][4];
  const int row_lo = warp * 16 + (lane >> 2);

  for (int t = 0; t < n_tiles; ++t) {
    if (t + 1 < n_tiles) load_tile(t + 1, (t + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) {
        const int row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = 2 * kk + (lane >> 4);
        ldsm_x4(sQa + swz<DH>(row, c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    const uint32_t kst = sKa + (t & 1) * kBN * DH * 2;
    const uint32_t vst = sVa + (t & 1) * kBN * DH * 2;

    // S = Q K^T : 16 rows x 64 keys per warp
    float sc[kBN / 8][4];
#pragma unroll
    for (int n = 0; n < kBN / 8; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < DH / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < kBN / 16; ++np) {
        uint32_t b0, b1, b2, b3;
        const int key = np * 16 + (lane & 7) + (lane >> 4) * 8;
        const int c = 2 * kk + ((lane >> 3) & 1);
        ldsm_x4(kst + swz<DH>(key, c), b0, b1, b2, b3);
        mma_bf16(sc[2 * np], qf[kk], b0, b1);
        mma_bf16(sc[2 * np + 1], qf[kk], b2, b3);
      }
    }

    // scale, mask, row max
    const int kbase = key0 + t * kBN;
    float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
    for (int n = 0; n < kBN / 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kl = n * 8 + (lane & 3) * 2 + (e & 1);  // key within tile
        const int key = kbase + kl;
        const int row = row_lo + (e >> 1) * 8;
        bool vis = key < key_end;
        if (tree_split && vis) vis = (sMask[row * 8 + (key >> 5)] >> (key & 31)) & 1u;
        const float v = vis ? sc[n][e] * p.scale_log2 : -INFINITY;
        sc[n][e] = v;
        if (e < 2) mx_lo = fmaxf(mx_lo, v);
        else mx_hi = fmaxf(mx_hi, v);
      }
    }
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
    const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
    const float base_lo = mn_lo == -INFINITY ? 0.f : mn_lo;
    const float base_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
    const float corr_lo = exp2f(m_lo - base_lo), corr_hi = exp2f(m_hi - base_hi);
    m_lo = mn_lo;
    m_hi = mn_hi;
    float sum_lo = 0.f, sum_hi = 0.f;
#pragma unroll
    for (int n = 0; n < kBN / 8; ++n) {
      sc[n][0] = exp2f(sc[n][0] - base_lo);
      sc[n][1] = exp2f(sc[n][1] - base_lo);
      sc[n][2] = exp2f(sc[n][2] - base_hi);
      sc[n][3] = exp2f(sc[n][3] - base_hi);
      sum_lo += sc[n][0] + sc[n][1];
      sum_hi += sc[n][2] + sc[n][3];
    }
    l_lo = l_lo * corr_lo + sum_lo;  // quad-partial sums; reduced at the end
    l_hi = l_hi * corr_hi + sum_hi;
#pragma unroll
    for (int n = 0; n < DH / 8; ++n) {
      o[n][0] *= corr_lo;
      o[n][1] *= corr_lo;
      o[n][2] *= corr_hi;
      o[n][3] *= corr_hi;
    }

    // O += P V with P = P_hi + P_lo
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk) {
      uint32_t ah[4], al[4];
      split_pair(sc[2 * kk][0], sc[2 * kk][1], ah[0], al[0]);
      split_pair(sc[2 * kk][2], sc[2 * kk][3], ah[1], al[1]);
      split_pair(sc[2 * kk + 1][0], sc[2 * kk + 1][1], ah[2], al[2]);
      split_pair(sc[2 * kk + 1][2], sc[2 * kk + 1][3], ah[3], al[3]);
#pragma unroll
      for (int np = 0; np < DH / 16; ++np) {
        uint32_t b0, b1, b2, b3;
        const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = 2 * np + (lane >> 4);
        ldsm_x4_t(vst + swz<DH>(key, c), b0, b1, b2, b3);
        mma_bf16(o[2 * np], ah, b0, b1);
        mma_bf16(o[2 * np + 1], ah, b2, b3);
        mma_bf16(o[2 * np], al, b0, b1);
        mma_bf16(o[2 * np + 1], al, b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);

  const size_t prow = ((size_t)bh * p.n_qt + qt) * p.S + s;  // partial block
  const float inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f;
  const float inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int row = row_lo + half * 8;
    if (qt * kBM + row >= p.R) continue;
    const float inv = half ? inv_hi : inv_lo;
    float* dst = p.o_part + (prow * kBM + row) * DH;
#pragma unroll
    for (int n = 0; n < DH / 8; ++n) {
      const int col = n * 8 + (lane & 3) * 2;
      float2 v;
      v.x = o[n][2 * half] * inv;
      v.y = o[n][2 * half + 1] * inv;
      *reinterpret_cast<float2*>(dst + col) = v;
    }
    if ((lane & 3) == 0) {
      const float m = half ? m_hi : m_lo;
      const float l = half ? l_hi : l_lo;
      p.lse_part[prow * kBM + row] = l > 0.f ? m + log2f(l) : -INFINITY;
    }
  }
}

// merge the splits of every query row; one warp per row
template <int DH>
__global__ void __launch_bounds__(256)
    attn_combine_kernel(AttnParams p, void* __restrict__ out, int out_f32) {
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int total = p.B * p.Hkv * p.R;
  if (gw >= total) return;
  const int bh = gw / p.R;
  const int r = gw - bh * p.R;
  const int b = bh / p.Hkv;
  const int kvh = bh - b * p.Hkv;
  const int P = p.prefix_len[b];
  if (P < 0 || P > p.max_prefix || P + p.N > p.cap) return;  // reported by the attention kernel
  const int n_split = (P + p.chunk - 1) / p.chunk + 1;
  const int qt = r / kBM, row = r - qt * kBM;
  const size_t pbase = ((size_t)bh * p.n_qt + qt) * p.S;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, p.lse_part[(pbase + s) * kBM + row]);
  constexpr int PER = DH / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const float lse = p.lse_part[(pbase + s) * kBM + row];
    const float w = lse == -INFINITY ? 0.f : exp2f(lse - M);
    wsum += w;
    const float* src = p.o_part + ((pbase + s) * kBM + row) * DH + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] += w * src[e];
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  const int node = r / p.G, g = r - node * p.G;
  const size_t obase = (((size_t)b * p.N + node) * p.Hq + kvh * p.G + g) * DH + lane * PER;
  if (out_f32) {
    float* o = static_cast<float*>(out) + obase;
#pragma unroll
    for (int e = 0; e < PER; ++e) o[e] = acc[e] * inv;
  } else {
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out) + obase;
#pragma unroll
    for (int e = 0; e < PER; ++e) o[e] = __float2bfloat16_rn(acc[e] * inv);
  }
}

// ----------------------------------------------------------------------------
// fp32 path
// ----------------------------------------------------------------------------
__global__ void tree_kv_write_f32_kernel(const float* __restrict__ k_new,
                                         const float* __restrict__ v_new, float* Kc, float* Vc,
                                         const int32_t* __restrict__ prefix_len, int B, int N,
                                         int Hkv, int dh, int cap, int max_prefix,
                                         int32_t* status) {
  const size_t total = (size_t)B * N * Hkv * dh;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int c = e % dh;
    const int kvh = (e / dh) % Hkv;
    const int j = (e / ((size_t)dh * Hkv)) % N;
    const int b = e / ((size_t)dh * Hkv * N);
    const int P = prefix_len[b];
    if (P < 0 || P > max_prefix || P + N > cap) {
      report(status, MEDUSA_ERR_DEVICE_CHECK);
      continue;
    }
    const size_t dst = (((size_t)b * Hkv + kvh) * cap + P + j) * dh + c;
    Kc[dst] = k_new[e];
    Vc[dst] = v_new[e];
  }
}

// one warp per (b, node, q head); lanes split dh
__global__ void __launch_bounds__(256)
    tree_attn_f32_kernel(const float* __restrict__ q, const float* __restrict__ k_new,
                         const float* __restrict__ v_new, const float* __restrict__ Kc,
                         const float* __restrict__ Vc, const int32_t* __restrict__ prefix_len,
                         const uint32_t* __restrict__ anc_mask, int B, int N, int Hq, int Hkv,
                         int dh, int cap, int max_prefix, int words, float scale, void* out,
                         int out_f32) {
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= B * N * Hq) return;
  const int hq = gw % Hq;
  const int i = (gw / Hq) % N;
  const int b = gw / (Hq * N);
  const int kvh = hq / (Hq / Hkv);
  const int P = prefix_len[b];
  if (P < 0 || P > max_prefix || P + N > cap) return;  // reported by the cache write
  constexpr int MAXPER = 8;
  const int per = dh / 32;
  float qv[MAXPER], acc[MAXPER];
  const float* qp = q + (size_t)gw * dh;
#pragma unroll
  for (int e = 0; e < MAXPER; ++e) {
    qv[e] = e < per ? qp[lane * per + e] : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  auto visit = [&](const float* kp, const float* vp) {
    float sdot = 0.f;
#pragma unroll
    for (int e = 0; e < MAXPER; ++e)
      if (e < per) sdot += qv[e] * kp[lane * per + e];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, o);
    const float sv = sdot * scale;
    const float mn = fmaxf(m, sv);
    const float corr = expf(m - mn);
    const float pw = expf(sv - mn);
    l = l * corr + pw;
#pragma unroll
    for (int e = 0; e < MAXPER; ++e)
      if (e < per) acc[e] = acc[e] * corr + pw * vp[lane * per + e];
    m = mn;
  };
  const size_t hb = ((size_t)b * Hkv + kvh) * cap;
  for (int t = 0; t < P; ++t) visit(Kc + (hb + t) * dh, Vc + (hb + t) * dh);
  for (int j = 0; j < N; ++j) {
    if ((anc_mask[(size_t)i * words + (j >> 5)] >> (j & 31)) & 1u) {
      const size_t off = (((size_t)b * N + j) * Hkv + kvh) * dh;
      visit(k_new + off, v_new + off);
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  if (out_f32) {
    float* o = static_cast<float*>(out) + (size_t)gw * dh;
#pragma unroll
    for (int e = 0; e < MAXPER; ++e)
      if (e < per) o[lane * per + e] = acc[e] * inv;
  } else {
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out) + (size_t)gw * dh;
#pragma unroll
    for (int e = 0; e < MAXPER; ++e)
      if (e < per) o[lane * per + e] = __float2bfloat16_rn(acc[e] * inv);
  }
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
namespace {

struct Split {
  int n_qt, S, chunk;
};

Split plan_split(int B, int N, int Hq, int Hkv, int max_prefix) {
  Split sp{};
  const int R = N * (Hq / Hkv);
  sp.n_qt = (R + kBM - 1) / kBM;
  const long long groups = (long long)B * Hkv * sp.n_qt;
  // about eight CTAs per SM of a 148-SM B200 (a fixed number, so that the
  // workspace size does not depend on the device queried)
  const long long target = 8LL * 148;
  long long splits = target / (groups > 0 ? groups : 1);
  if (splits < 1) splits = 1;
  int chunk = (int)((max_prefix + splits - 1) / splits);
  chunk = ((chunk + kBN - 1) / kBN) * kBN;
  if (chunk < 4 * kBN) chunk = 4 * kBN;
  sp.chunk = chunk;
  sp.S = (max_prefix + chunk - 1) / chunk + 1;
  return sp;
}

template <int DH>
size_t attn_smem() {
  return (size_t)kBM * DH * 2 + 4 * (size_t)kBN * DH * 2 + kBM * 8 * 4;
}

}  // namespace

size_t tree_attention_workspace_size(int B, int N, int Hq, int Hkv, int dh, int max_prefix,
                                     medusa_dtype_t dt) {
  if (dt == MEDUSA_F32) return 0;
  const Split sp = plan_split(B, N, Hq, Hkv, max_prefix);
  const size_t rows = (size_t)B * Hkv * sp.n_qt * sp.S * kBM;
  return align256(rows * dh * 4) + align256(rows * 4);
}

template <int DH>
static medusa_status_t launch_bf16(AttnParams& p, void* out, int out_f32, cudaStream_t stream) {
  const size_t smem = attn_smem<DH>();
  if (cudaFuncSetAttribute(tree_attn_bf16_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return fail(MEDUSA_ERR_CUDA, "cudaFuncSetAttribute(tree_attention) failed");
  dim3 grid(p.S, p.n_qt, p.B * p.Hkv);
  tree_attn_bf16_kernel<DH><<<grid, kAttnThreads, smem, stream>>>(p);
  medusa_status_t st = check_launch("tree_attention");
  if (st != MEDUSA_OK) return st;
  const int rows = p.B * p.Hkv * p.R;
  attn_combine_kernel<DH><<<(rows + 7) / 8, 256, 0, stream>>>(p, out, out_f32);
  return check_launch("tree_attention_combine");
}

medusa_status_t tree_attention(const void* q, const void* k_new, const void* v_new, void* Kc,
                               void* Vc, const int32_t* prefix_len, const uint32_t* anc_mask,
                               medusa_dtype_t dt, int B, int N, int Hq, int Hkv, int dh, int cap,
                               int max_prefix, float scale, void* out, medusa_dtype_t out_dt,
                               void* ws, int32_t* status, cudaStream_t stream) {
  const int words = (N + 31) / 32;
  const int out_f32 = out_dt == MEDUSA_F32 ? 1 : 0;
  if (dt == MEDUSA_F32) {
    const size_t total = (size_t)B * N * Hkv * dh;
    const int blocks = (int)((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
    tree_kv_write_f32_kernel<<<blocks, 256, 0, stream>>>(
        static_cast<const float*>(k_new), static_cast<const float*>(v_new),
        static_cast<float*>(Kc), static_cast<float*>(Vc), prefix_len, B, N, Hkv, dh, cap,
        max_prefix, status);
    medusa_status_t st = check_launch("tree_kv_write_f32");
    if (st != MEDUSA_OK) return st;
    const int rows = B * N * Hq;
    tree_attn_f32_kernel<<<(rows + 7) / 8, 256, 0, stream>>>(
        static_cast<const float*>(q), static_cast<const float*>(k_new),
        static_cast<const float*>(v_new), static_cast<const float*>(Kc),
        static_cast<const float*>(Vc), prefix_len, anc_mask, B, N, Hq, Hkv, dh, cap, max_prefix,
        words, scale, out, out_f32);
    return check_launch("tree_attention_f32");
  }
  const Split sp = plan_split(B, N, Hq, Hkv, max_prefix);
  AttnParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.Kc = static_cast<__nv_bfloat16*>(Kc);
  p.Vc = static_cast<__nv_bfloat16*>(Vc);
  p.prefix_len = prefix_len;
  p.anc_mask = anc_mask;
  const size_t rows = (size_t)B * Hkv * sp.n_qt * sp.S * kBM;
  p.o_part = static_cast<float*>(ws);
  p.lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + align256(rows * dh * 4));
  p.B = B;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.R = N * p.G;
  p.n_qt = sp.n_qt;
  p.S = sp.S;
  p.chunk = sp.chunk;
  p.cap = cap;
  p.max_prefix = max_prefix;
  p.words = words;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = status;
  if (dh == 128) return launch_bf16<128>(p, out, out_f32, stream);
  return launch_bf16<64>(p, out, out_f32, stream);
}

}  // namespace medusa
