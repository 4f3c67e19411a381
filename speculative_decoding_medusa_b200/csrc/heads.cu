// Medusa heads + per-head top-k.
//
// "Medusa Heads" glossary, "Comment les têtes prédisent les tokens suivants":
// head k = h + SiLU(W1_k h + b1_k), then a projection W2_k to the vocabulary.
//
// bf16 path: two launches of one weight-streaming tcgen05 GEMM and a merge.
//   1. W1 stage: U = W1 * h^T (rows = K*d output features, columns = batch).
//      Epilogue: y = h + SiLU(U + b1), written as two bf16 rows (hi, lo) per
//      sequence into Y [K, 2B, d] so that y enters the next GEMM at ~16-bit
//      mantissa precision.
//   2. W2 stage: Z = W2 * Y^T (rows = K*V tokens, columns = 2B); the epilogue
//      adds the hi/lo columns, optionally stores the fp32 logits, sorts every
//      32-row slice (warp bitonic sort) and merges them into the tile's best
//      list, which joins a running best list per (head, sequence) that the
//      CTA keeps in shared memory across its tiles (one list per tile when
//      those lists do not fit).  Tiles are handed out by an atomic counter.
//   3. topk_merge: per (sequence, head), the best kmax of all the lists;
//      when a tree is given, the cluster that completes a sequence's K lists
//      also builds that sequence's candidate tree.
// The weights are the only large operand (K*(d^2 + V*d) bf16): every CTA
// streams 128-row weight tiles through a TMA -> shared memory -> tcgen05.mma
// pipeline; the batch sits in the MMA's N dimension (weight rows fill M=128).
// The first GEMM's few tiles are split evenly by k-blocks over the CTAs
// (stream-K) when whole tiles would leave SMs idle.
//
// fp32 path (small shapes): warp-per-row CUDA-core dot products, same merge.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <cooperative_groups.h>

#include "abi_internal.h"
#include "common.cuh"
#include "tree_build.cuh"

namespace cg = cooperative_groups;

namespace medusa {

// ----------------------------------------------------------------------------
// weight-streaming GEMM on tcgen05
// ----------------------------------------------------------------------------

constexpr int kTileM = 128;  // weight rows per tile = UMMA M
constexpr int kTileK = 64;   // bf16 elements per 128-byte swizzled row
constexpr int kGemmThreads = 192;

enum GemmMode { kModeW1 = 0, kModeW2 = 1 };

struct GemmParams {
  int rows_per_head;  // d (W1) or V (W2)
  int n_heads;        // K
  int d;              // reduction length
  int B;              // sequences
  int tiles_per_head;
  int n_tiles;
  int b_head_stride;  // 0: one B operand for all heads (W1), 1: per head (W2)
  int kmax;
  const __nv_bfloat16* h;     // [B, d] (W1 epilogue)
  const __nv_bfloat16* b1;    // [K, d] (W1 epilogue)
  __nv_bfloat16* Y;           // [K, 2B, d] (W1 epilogue output)
  float* logits;              // [B, K, V] or null (W2 epilogue)
  float* part_vals;           // [B*K, tiles_per_head, kmax] (W2)
  int32_t* part_ids;
  int32_t* status;
  // stream-K (W1 mode): every CTA takes kpc consecutive k-blocks of the
  // (tile, k-block) sequence; 0 = whole tiles round-robin
  int kpc;
  float* sk_part;  // [grid][kTileM][NB] fp32 partial of a CTA's leading tile tail
  int* sk_flag;    // [grid] 1 once that partial is written (zeroed by a kernel before the launch)
  int sk_grid;     // CTAs of a stream-K launch
  // second GEMM: tiles handed out by this counter (tiles past the first
  // grid-full are claimed one at a time); the first GEMM zeroes it.  Null:
  // whole tiles round-robin.
  int* tile_counter;
  // second GEMM: 1 = each CTA keeps a best-32 list per (head, sequence) in
  // shared memory across its tiles and writes one list per row at the end
  // (list blockIdx.x of gridDim.x); 0 = one list per tile (list tile_in_head)
  int run_lists;
};

// tile ids a CTA's producer has claimed and not every role has read yet: the
// producer runs at most S stages ahead of the MMA issuer, which runs at most
// two tiles ahead of the epilogue, so S + 3 <= 11 slots are ever in use
constexpr int kTileRing = 16;

// One CTA's work as (tile, first k-block, end k-block) segments, in order.
// Round-robin: whole tiles blockIdx.x, + gridDim.x, ...  Stream-K: the
// k-blocks [blockIdx.x * kpc, + kpc) of the tile-major sequence, cut at tile
// ends; only the first segment can start inside a tile.  Dynamic (whole
// tiles): tile blockIdx.x first, then tiles gridDim.x + (counter++) until
// they run out, so that CTAs which stream faster take more tiles; the
// producer claims each tile and publishes it in a ring slot with its own
// mbarrier, which the MMA issuer and the epilogue wait on before reading it.
struct SegIter {
  int nkb, n_tiles, kpc, tile, g, g_hi;
  int* counter;        // dynamic mode when set
  int* ring;           // [kTileRing] tile ids
  uint64_t* ring_bar;  // [kTileRing]
  bool producer;
  int it;
  volatile int* abort;
  int32_t* status;
  __device__ __forceinline__ void init(const GemmParams& p, int nkb_, int* counter_ = nullptr,
                                       int* ring_ = nullptr, uint64_t* ring_bar_ = nullptr,
                                       bool producer_ = false, volatile int* abort_ = nullptr) {
    nkb = nkb_;
    n_tiles = p.n_tiles;
    kpc = p.kpc;
    tile = blockIdx.x;
    g = blockIdx.x * kpc;
    g_hi = min(g + kpc, n_tiles * nkb);
    counter = counter_;
    ring = ring_;
    ring_bar = ring_bar_;
    producer = producer_;
    it = 0;
    abort = abort_;
    status = p.status;
  }
  __device__ __forceinline__ bool next(int& t, int& kb0, int& kb1) {
    if (counter != nullptr) {
      const int slot = it % kTileRing;
      if (producer) {
        t = it == 0 ? static_cast<int>(blockIdx.x)
                    : static_cast<int>(gridDim.x) + atomicAdd(counter, 1);
        ring[slot] = t;
        mbar_arrive(&ring_bar[slot]);  // release: the id is visible to its waiters
      } else {
        if (!mbar_wait_bounded(&ring_bar[slot], (it / kTileRing) & 1, abort, status)) return false;
        t = ring[slot];
      }
      ++it;
      kb0 = 0;
      kb1 = nkb;
      return t < n_tiles;
    }
    if (kpc > 0) {
      if (g >= g_hi) return false;
      t = g / nkb;
      kb0 = g - t * nkb;
      kb1 = min(nkb, kb0 + (g_hi - g));
      g += kb1 - kb0;
      return true;
    }
    if (tile >= n_tiles) return false;
    t = tile;
    kb0 = 0;
    kb1 = nkb;
    tile += gridDim.x;
    return true;
  }
};

template <int NB, int S>
struct GemmSmem {
  static constexpr int kABytes = kTileM * kTileK * 2;  // 16 KB
  static constexpr int kBBytes = NB * kTileK * 2;
  static constexpr int kStageTx = kABytes + kBBytes;
  static constexpr int kAOff = 0;
  static constexpr int kBOff = S * kABytes;
  static constexpr int kBarOff = kBOff + S * kBBytes;
  // full[S], empty[S], tfull[2], tempty[2], drain, epilogue, ring[kTileRing], exit
  static constexpr int kNumBars = 2 * S + 7 + kTileRing;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kRingOff = kMiscOff + 16;  // [kTileRing] claimed tile ids
  // per-warp sorted lists of the W2 epilogue: [4 quads][8 sequences][32] (value, index)
  static constexpr int kListOff = kRingOff + kTileRing * 4;
  static constexpr int kListBytes = 4 * 8 * 32 * 8;
  static constexpr int kBytes = kListOff + kListBytes;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base
  // running lists (second GEMM, run_lists): [K*B][32] values, then ids,
  // after kBytes; K*B*256 bytes more at launch
};

// a (head, sequence) row's running list takes 32 values and 32 ids
constexpr int kRunRowBytes = 32 * 8;
constexpr int kRunMaxRows = 128;  // K * B up to which the running lists are used
constexpr int kSmemLimit = 227 * 1024;

template <int NB>
__host__ __device__ constexpr uint32_t tmem_cols() {
  return (2 * NB) < 32 ? 32u : static_cast<uint32_t>(2 * NB);
}

template <int NB, int S, int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    heads_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, GemmParams p) {
  grid_dep_wait();
  grid_dep_launch();
  // the first GEMM resets the second GEMM's tile counter (the second GEMM
  // reads it only after waiting for this kernel)
  // (and the merge's per-sequence row counts that follow it)
  if (MODE == kModeW1 && p.tile_counter != nullptr && blockIdx.x == 0 && threadIdx.x <= p.B)
    p.tile_counter[threadIdx.x] = 0;
  using L = GemmSmem<NB, S>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + 2;
  uint64_t* drain = bars + 2 * S + 4;
  uint64_t* epi = bars + 2 * S + 5;
  uint64_t* ring_bar = bars + 2 * S + 6;
  uint64_t* exit_bar = ring_bar + kTileRing;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  int* ring = reinterpret_cast<int*>(smem + L::kRingOff);
  // the second GEMM hands out tiles dynamically when given a counter
  int* const dyn_counter = MODE == kModeW2 ? p.tile_counter : nullptr;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nkb = p.d / kTileK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    mbar_init(epi, 128);
    for (int i = 0; i < kTileRing; ++i) mbar_init(&ring_bar[i], 1);
    mbar_init(exit_bar, kGemmThreads);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, tmem_cols<NB>());
    tmem_relinquish();
  }
  tc_fence_before();
  // every warp reconverges first: lane 0 of some warps ran a role alone
  __syncwarp();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      const uint64_t pol_a = l2_policy_evict_first();
      const uint64_t pol_b = l2_policy_evict_last();
      int g = 0;
      bool ok = true;
      SegIter seg;
      seg.init(p, nkb, dyn_counter, ring, ring_bar, true, abort_flag);
      int tile, kb0, kb1;
      while (ok && seg.next(tile, kb0, kb1)) {
        const int head = tile / p.tiles_per_head;
        const int m0 = (tile - head * p.tiles_per_head) * kTileM;
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
          const int s = g % S;
          const uint32_t ph = (g / S) & 1;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], L::kStageTx);
          tma_load_3d(smem + L::kAOff + s * L::kABytes, &tmA, &full[s], kb * kTileK, m0, head,
                      pol_a);
          tma_load_3d(smem + L::kBOff + s * L::kBBytes, &tmB, &full[s], kb * kTileK, 0,
                      head * p.b_head_stride, pol_b);
        }
      }
      // let every copy this thread issued land before the CTA can exit
      const int first = g > S ? g - S : 0;
      for (int x = first; x < g; ++x) {
        int dummy_abort = 0;
        mbar_wait_bounded(&full[x % S], (x / S) & 1, &dummy_abort, p.status);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kTileM, NB);
      int g = 0, it = 0;
      bool ok = true;
      SegIter seg;
      seg.init(p, nkb, dyn_counter, ring, ring_bar, false, abort_flag);
      int tile, kb0, kb1;
      for (; ok && seg.next(tile, kb0, kb1); ++it) {
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[acc], aph ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * NB;
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
          const int s = g % S;
          const uint32_t ph = (g / S) & 1;
          if (!mbar_wait_bounded(&full[s], ph, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + L::kAOff + s * L::kABytes);
          const uint32_t b_addr = smem_u32(smem + L::kBOff + s * L::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk) {
            umma_bf16(d_tmem, umma_desc_sw128(a_addr + kk * 32), umma_desc_sw128(b_addr + kk * 32),
                      idesc, (kb > kb0 || kk != 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      // every MMA this thread issued must finish before TMEM is released
      umma_commit(drain);
      int dummy_abort = 0;
      mbar_wait_bounded(drain, 0, &dummy_abort, p.status);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;
    // the four epilogue warps synchronise on an mbarrier with a bounded wait,
    // so that one warp giving up cannot leave the others blocked
    uint32_t epi_phase = 0;
    bool epi_ok = true;
    auto epi_sync = [&]() {
      mbar_arrive(epi);
      epi_ok = mbar_wait_bounded(epi, epi_phase, abort_flag, p.status);
      epi_phase ^= 1u;
      return epi_ok;
    };
    // running lists of the second GEMM: warp quad owns the sequences b with
    // b % 4 == quad (the warp that merges them in every tile below), so a
    // row's list is only ever touched by one warp
    const bool run = MODE == kModeW2 && p.run_lists != 0;
    const int run_rows = p.n_heads * p.B;
    float* run_v = reinterpret_cast<float*>(smem + L::kBytes);
    int* run_i = reinterpret_cast<int*>(smem + L::kBytes + (size_t)run_rows * 32 * 4);
    if (run) {
      for (int e = threadIdx.x - 64; e < run_rows * 32; e += 128) {
        run_v[e] = -INFINITY;
        run_i[e] = 0x7fffffff;
      }
      epi_sync();
    }
    int it = 0;
    SegIter seg;
    seg.init(p, nkb, dyn_counter, ring, ring_bar, false, abort_flag);
    int tile, kb0, kb1;
    for (; epi_ok && seg.next(tile, kb0, kb1); ++it) {
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      const int head = tile / p.tiles_per_head;
      const int tile_in_head = tile - head * p.tiles_per_head;
      const int r = tile_in_head * kTileM + row;  // row within the head
      const bool valid = r < p.rows_per_head;
      // The first GEMM's epilogue inputs (bias, residual h of the first 16
      // sequences) do not depend on the MMA: their loads are issued before
      // the wait for it.
      float pre_bias = 0.f;
      float pre_h[16];
      if (MODE == kModeW1 && kb0 == 0 && valid) {
        pre_bias = __bfloat162float(p.b1[(size_t)head * p.d + r]);
#pragma unroll
        for (int t = 0; t < 16; ++t)
          pre_h[t] = t < p.B ? __bfloat162float(p.h[(size_t)t * p.d + r]) : 0.f;
      }
      if (!mbar_wait_bounded(&tfull[acc], aph, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * NB;
      if (MODE == kModeW1 && kb0 > 0) {
        // stream-K: the tail of a tile that an earlier CTA finishes.  This
        // CTA's fp32 partial goes to its slot, then its flag is raised.
        float* dst = p.sk_part + ((size_t)blockIdx.x * kTileM + row) * NB;
#pragma unroll 1
        for (int c0 = 0; c0 < NB; c0 += 16) {
          float v[16];
          tmem_ld16(taddr + c0, v);
#pragma unroll
          for (int t = 0; t < 16; t += 4)
            *reinterpret_cast<float4*>(dst + c0 + t) = make_float4(v[t], v[t + 1], v[t + 2], v[t + 3]);
        }
        __threadfence();
        if (!epi_sync()) break;
        if (threadIdx.x == 64) st_release_gpu(&p.sk_flag[blockIdx.x], 1);
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        continue;
      }
      // stream-K: this CTA holds the tile's first k-block; the CTAs after it
      // that took the rest have written their partials
      int c_last = blockIdx.x;
      if (MODE == kModeW1 && kb1 < nkb) {
        c_last = ((tile + 1) * nkb - 1) / p.kpc;
        bool ready = true;
        for (int c = blockIdx.x + 1; ready && c <= c_last; ++c)
          ready = wait_flag_bounded(&p.sk_flag[c], 1, abort_flag, p.status, kSpinBudgetCycles);
        if (!ready) break;
      }
#pragma unroll 1
      for (int c0 = 0; epi_ok && c0 < NB; c0 += 16) {
        float v[16];
        tmem_ld16(taddr + c0, v);
        for (int c = blockIdx.x + 1; c <= c_last; ++c) {
          const float* src = p.sk_part + ((size_t)c * kTileM + row) * NB + c0;
#pragma unroll
          for (int t = 0; t < 16; t += 4) {
            const float4 q = *reinterpret_cast<const float4*>(src + t);
            v[t] += q.x;
            v[t + 1] += q.y;
            v[t + 2] += q.z;
            v[t + 3] += q.w;
          }
        }
        if (MODE == kModeW1) {
          if (valid) {
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              const int b = c0 + t;
              if (b < p.B) {
                const float u = v[t] + pre_bias;
                const float hb = c0 == 0 ? pre_h[t] : __bfloat162float(p.h[(size_t)b * p.d + r]);
                const float y = hb + u / (1.0f + expf(-u));
                const __nv_bfloat16 hi = __float2bfloat16_rn(y);
                const __nv_bfloat16 lo = __float2bfloat16_rn(y - __bfloat162float(hi));
                const size_t base = ((size_t)head * 2 * p.B + 2 * b) * p.d + r;
                p.Y[base] = hi;
                p.Y[base + p.d] = lo;
              }
            }
          }
        } else {
          float* lv = reinterpret_cast<float*>(smem + L::kListOff);
          int* li = reinterpret_cast<int*>(smem + L::kListOff + 4 * 8 * 32 * 4);
          // each warp sorts its 32 rows per sequence ...
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int b = (c0 >> 1) + t;
            if (b >= p.B) continue;  // uniform across the warp
            const float z = v[2 * t] + v[2 * t + 1];
            const size_t row_bk = (size_t)b * p.n_heads + head;
            if (p.logits != nullptr && valid) p.logits[row_bk * p.rows_per_head + r] = z;
            float sv = valid ? z : -INFINITY;
            int si = valid ? r : 0x7fffffff;
            warp_sort_desc(sv, si);
            lv[(quad * 8 + t) * 32 + lane] = sv;
            li[(quad * 8 + t) * 32 + lane] = si;
          }
          if (!epi_sync()) break;
          // ... then warp `quad` merges the four lists of sequences quad, quad+4
#pragma unroll
          for (int t = quad; t < 8; t += 4) {
            const int b = (c0 >> 1) + t;
            if (b >= p.B) continue;
            float rv = lv[t * 32 + lane];
            int ri = li[t * 32 + lane];
#pragma unroll
            for (int q2 = 1; q2 < 4; ++q2)
              warp_merge_top32(rv, ri, lv[(q2 * 8 + t) * 32 + lane], li[(q2 * 8 + t) * 32 + lane]);
            if (run) {
              const int at = (head * p.B + b) * 32 + lane;
              warp_merge_top32(rv, ri, run_v[at], run_i[at]);
              run_v[at] = rv;
              run_i[at] = ri;
            } else if (lane < p.kmax) {
              const size_t row_bk = (size_t)b * p.n_heads + head;
              const size_t o = (row_bk * p.tiles_per_head + tile_in_head) * p.kmax + lane;
              p.part_vals[o] = rv;
              p.part_ids[o] = ri;
            }
          }
          if (!epi_sync()) break;
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
    // one list per (sequence, head) row: list blockIdx.x of gridDim.x
    if (run && epi_ok) {
      for (int rr = 0; rr < run_rows; ++rr) {
        const int head = rr / p.B, b = rr - head * p.B;
        if ((b & 3) != quad) continue;  // the warp that owns the row
        if (lane < p.kmax) {
          const size_t o = (((size_t)b * p.n_heads + head) * gridDim.x + blockIdx.x) * p.kmax + lane;
          p.part_vals[o] = run_v[rr * 32 + lane];
          p.part_ids[o] = run_i[rr * 32 + lane];
        }
      }
    }
  }

  // TMEM is released once every thread is past its last TMEM access: each
  // thread arrives on the exit barrier (an mbarrier counts threads, however
  // the warps' lanes diverged in their roles) and warp 1 waits for all.
  tc_fence_before();
  mbar_arrive(exit_bar);
  if (warp == 1) {
    // lanes 1..31 wait here, parked, until the MMA thread (lane 0) is done:
    // spinning on the barrier beside it would take its issue slots
    __syncwarp();
    int no_abort = 0;
    mbar_wait_bounded(exit_bar, 0, &no_abort, p.status);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols<NB>());
  }
}

// The first GEMM's stream-K flags, cleared before each call by a kernel (so
// that the launches stay chained by programmatic dependent launch, which a
// memset node would break).
__global__ void __launch_bounds__(256) heads_flags_zero_kernel(int* __restrict__ flags, int n) {
  grid_dep_wait();
  grid_dep_launch();
  for (int e = threadIdx.x; e < n; e += blockDim.x) flags[e] = 0;
}

// ----------------------------------------------------------------------------
// top-k merge: best kmax of C candidates per row
//
// A row is shared by a cluster of kMergeCtas CTAs of kMergeWarps warps: warp w
// of CTA r walks the candidate chunks (w * kMergeCtas + r) * 32, + 32 * all
// warps, keeping a sorted best-32 list filtered by its kmax-th entry.  The
// warps of a CTA merge pairwise through shared memory (three rounds), then CTA
// 0 of the cluster reads the other CTAs' lists from distributed shared memory
// and merges them.
// ----------------------------------------------------------------------------
// Candidates of row r: C = n_lists * list_len entries; entry e is list
// g = e / list_len, position j = e % list_len, stored at r * row_stride +
// g * list_stride + j, and its id gains id_offsets[g] when id_offsets is set.
// (The heads' own tile lists are one list of C contiguous entries per row.)
struct MergeLayout {
  long long row_stride, list_stride;
  int list_len;
  const int32_t* id_offsets;
};

constexpr int kMergeWarps = 8;
constexpr int kMergeCtas = 8;    // cluster size (portable)
constexpr int kMergeUnroll = 2;  // 32-candidate chunks each warp has in flight
static_assert(kMergeWarps * 32 == kTreeThreads, "the merge's tail builds trees with its CTA");

// The tree built by the merge's tail: rows are (sequence, head) pairs, row =
// b * tree.K + head; seq_count[b] counts sequence b's finished rows (zero
// before the launch).  tree.cand_ids == nullptr: no tail.
struct MergeTree {
  TreeOut tree;
  int* seq_count;
};

__global__ void __cluster_dims__(kMergeCtas, 1, 1) __launch_bounds__(kMergeWarps * 32)
    topk_merge_kernel(const float* __restrict__ vals, const int32_t* __restrict__ ids, long long C,
                      int kmax, int32_t* __restrict__ out_ids, float* __restrict__ out_vals,
                      MergeLayout lay, MergeTree mt) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ float sv[kMergeWarps][32];
  __shared__ int si[kMergeWarps][32];
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const long long row = blockIdx.x / kMergeCtas;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const size_t base = (size_t)row * lay.row_stride;
  constexpr long long kStride = (long long)kMergeCtas * kMergeWarps * 32 * kMergeUnroll;
  // running best-32 of this warp, sorted, and its kmax-th entry as a filter
  float rv = -INFINITY;
  int ri = 0x7fffffff;
  float tv = -INFINITY;
  int ti = 0x7fffffff;
  for (long long c = (long long)(warp * kMergeCtas + crank) * 32 * kMergeUnroll; c < C;
       c += kStride) {
    float v[kMergeUnroll];
    int i[kMergeUnroll];
#pragma unroll
    for (int u = 0; u < kMergeUnroll; ++u) {
      const long long e = c + u * 32 + lane;
      v[u] = -INFINITY;
      i[u] = 0x7fffffff;
      if (e < C) {
        const int g = static_cast<int>(e / lay.list_len);
        const size_t at = base + (size_t)g * lay.list_stride + (e - (long long)g * lay.list_len);
        v[u] = vals[at];
        i[u] = ids != nullptr ? ids[at] : static_cast<int>(e);
        if (lay.id_offsets != nullptr) i[u] += lay.id_offsets[g];
      }
    }
#pragma unroll
    for (int u = 0; u < kMergeUnroll; ++u) {
      if (__any_sync(0xffffffffu, better(v[u], i[u], tv, ti))) {
        warp_sort_desc(v[u], i[u]);
        warp_merge_top32(rv, ri, v[u], i[u]);
        tv = __shfl_sync(0xffffffffu, rv, kmax - 1);
        ti = __shfl_sync(0xffffffffu, ri, kmax - 1);
      }
    }
  }
  // warps of the CTA: pairwise rounds
  sv[warp][lane] = rv;
  si[warp][lane] = ri;
#pragma unroll
  for (int s = kMergeWarps / 2; s > 0; s >>= 1) {
    __syncthreads();
    if (warp < s) {
      warp_merge_top32(rv, ri, sv[warp + s][lane], si[warp + s][lane]);
      sv[warp][lane] = rv;
      si[warp][lane] = ri;
    }
  }
  // CTAs of the cluster: CTA 0 merges the others' lists (row 0 of their sv/si)
  cluster.sync();
  if (crank == 0 && warp == 0) {
    for (int r = 1; r < kMergeCtas; ++r) {
      const float* rsv = cluster.map_shared_rank(&sv[0][0], r);
      const int* rsi = cluster.map_shared_rank(&si[0][0], r);
      warp_merge_top32(rv, ri, rsv[lane], rsi[lane]);
    }
    if (lane < kmax) {
      out_ids[(size_t)row * kmax + lane] = ri;
      out_vals[(size_t)row * kmax + lane] = rv;
    }
  }
  if (mt.tree.cand_ids != nullptr && crank == 0) {
    // Count this row in.  The CTA whose row completes sequence b's K lists
    // builds b's candidate tree from them; no CTA waits for another.
    __shared__ int s_last;
    const int b = static_cast<int>(row / mt.tree.K);
    if (warp == 0) {
      __threadfence();  // this lane's list entry before the count
      __syncwarp();
      if (lane == 0) s_last = atomicAdd(&mt.seq_count[b], 1) == mt.tree.K - 1;
      __syncwarp();
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      const int32_t* lists = out_ids + (size_t)b * mt.tree.K * kmax;
      build_tree_sequence(mt.tree, b, [lists](int e) { return __ldcg(lists + e); }, b == 0);
    }
  }
  // no CTA leaves while CTA 0 may still read its shared memory
  cluster.sync();
}

// ----------------------------------------------------------------------------
// fp32 CUDA-core path
// ----------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// y[b][k][j] = h[b][j] + SiLU(W1[k][j] . h[b] + b1[k][j]); one warp per j.
__global__ void __launch_bounds__(256)
    heads_f32_w1_kernel(const float* __restrict__ h, const float* __restrict__ W1,
                        const float* __restrict__ b1, int B, int d, int K, float* __restrict__ y,
                        int* __restrict__ seq_count) {
  grid_dep_wait();
  grid_dep_launch();
  // the merge's per-sequence row counts
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < B) seq_count[threadIdx.x] = 0;
  const int k = blockIdx.y;
  const int j = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (j >= d) return;
  const float* w = W1 + ((size_t)k * d + j) * d;
  for (int b = 0; b < B; ++b) {
    float s = 0.f;
    for (int e = lane; e < d; e += 32) s += w[e] * h[(size_t)b * d + e];
    s = warp_sum(s);
    if (lane == 0) {
      const float u = s + b1[(size_t)k * d + j];
      y[((size_t)b * K + k) * d + j] = h[(size_t)b * d + j] + u / (1.0f + expf(-u));
    }
  }
}

// z[b][k][v] = W2[k][v] . y[b][k]; one warp per v.
__global__ void __launch_bounds__(256)
    heads_f32_w2_kernel(const float* __restrict__ y, const float* __restrict__ W2, int B, int d,
                        int V, int K, float* __restrict__ z) {
  grid_dep_wait();
  grid_dep_launch();
  const int k = blockIdx.y;
  const int v = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (v >= V) return;
  const float* w = W2 + ((size_t)k * V + v) * d;
  for (int b = 0; b < B; ++b) {
    const float* yy = y + ((size_t)b * K + k) * d;
    float s = 0.f;
    for (int e = lane; e < d; e += 32) s += w[e] * yy[e];
    s = warp_sum(s);
    if (lane == 0) z[((size_t)b * K + k) * V + v] = s;
  }
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
medusa_status_t topk_merge_lists(const float* vals, const int32_t* ids, int rows, int n_lists,
                                 int list_len, long long row_stride, long long list_stride,
                                 const int32_t* id_offsets, int kmax, int32_t* out_ids,
                                 float* out_vals, cudaStream_t stream) {
  const MergeLayout lay{row_stride, list_stride, list_len, id_offsets};
  launch(topk_merge_kernel, rows * kMergeCtas, kMergeWarps * 32, 0, stream, vals, ids,
         (long long)n_lists * list_len, kmax, out_ids, out_vals, lay, MergeTree{});
  return check_launch("topk_merge");
}

namespace {

// bf16 tensor [dim2][dim1][dim0] (dim0 contiguous), box {64, box1, 1}
bool make_map_3d(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                 uint32_t box1) {
  const uint64_t dims[3] = {dim0, dim1, dim2};
  const uint64_t strides[2] = {dim0 * 2, dim0 * dim1 * 2};
  const uint32_t box[3] = {static_cast<uint32_t>(kTileK), box1, 1};
  return make_tmap_bf16(map, base, 3, dims, strides, box);
}

int num_sms() { return device_sm_count(); }

int gemm_grid(const GemmParams& p) {
  return p.kpc > 0 ? p.sk_grid : (p.n_tiles < num_sms() ? p.n_tiles : num_sms());
}

template <int NB, int S, int MODE>
medusa_status_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p,
                            cudaStream_t stream) {
  using L = GemmSmem<NB, S>;
  auto kern = heads_gemm_kernel<NB, S, MODE>;
  const size_t smem =
      L::kAlloc + (p.run_lists ? (size_t)p.n_heads * p.B * kRunRowBytes : (size_t)0);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return fail(MEDUSA_ERR_CUDA, "cudaFuncSetAttribute(heads_gemm) failed");
  launch(kern, gemm_grid(p), kGemmThreads, smem, stream, a, b, p);
  return check_launch("heads_gemm");
}

// shared memory of the GEMM at width nb before any running lists
size_t gemm_alloc_bytes(int nb) {
  switch (nb) {
    case 16: return GemmSmem<16, 8>::kAlloc;
    case 32: return GemmSmem<32, 8>::kAlloc;
    case 64: return GemmSmem<64, 8>::kAlloc;
    case 128: return GemmSmem<128, 4>::kAlloc;
    case 256: return GemmSmem<256, 3>::kAlloc;
  }
  return 0;
}

template <int MODE>
medusa_status_t launch_gemm_nb(int nb, const CUtensorMap& a, const CUtensorMap& b,
                               const GemmParams& p, cudaStream_t s) {
  switch (nb) {
    case 16: return launch_gemm<16, 8, MODE>(a, b, p, s);
    case 32: return launch_gemm<32, 8, MODE>(a, b, p, s);
    case 64: return launch_gemm<64, 8, MODE>(a, b, p, s);  // 128 KB of weights in flight
    case 128: return launch_gemm<128, 4, MODE>(a, b, p, s);
    case 256: return launch_gemm<256, 3, MODE>(a, b, p, s);
  }
  return fail(MEDUSA_ERR_UNSUPPORTED, "heads: unsupported MMA width");
}

int round_nb(int cols) {
  int nb = 16;
  while (nb < cols) nb *= 2;
  return nb;
}

struct HeadsWs {
  size_t y_bytes, part_bytes, sk_part_bytes, sk_flag_bytes, counter_bytes, total;
};

HeadsWs heads_ws_layout(int B, int d, int V, int K, int kmax, medusa_dtype_t dt) {
  HeadsWs w{};
  if (dt == MEDUSA_BF16) {
    const size_t tph = (size_t)(V + kTileM - 1) / kTileM;
    w.y_bytes = align256((size_t)K * 2 * B * d * 2);
    // candidate lists per row: one per tile, or one per CTA (running lists)
    const size_t lists = tph > (size_t)num_sms() ? tph : (size_t)num_sms();
    w.part_bytes = align256((size_t)B * K * lists * kmax * 4);
    // stream-K partials of the first GEMM: one [128][NB] fp32 slot and one
    // flag per CTA
    w.sk_part_bytes = align256((size_t)num_sms() * kTileM * round_nb(B) * 4);
    w.sk_flag_bytes = align256((size_t)num_sms() * 4);
    // the second GEMM's tile counter, then the merge's row count per sequence
    w.counter_bytes = align256((size_t)(B + 1) * 4);
    w.total = w.y_bytes + 2 * w.part_bytes + w.sk_part_bytes + w.sk_flag_bytes + w.counter_bytes;
  } else {
    w.y_bytes = align256((size_t)B * K * d * 4);
    w.part_bytes = align256((size_t)B * K * V * 4);
    w.counter_bytes = align256((size_t)B * 4);  // the merge's row count per sequence
    w.total = w.y_bytes + w.part_bytes + w.counter_bytes;
  }
  return w;
}

}  // namespace

size_t heads_topk_workspace_size(int B, int d, int V, int K, int kmax, medusa_dtype_t dt) {
  return heads_ws_layout(B, d, V, K, kmax, dt).total;
}

medusa_status_t heads_topk(const void* h, const void* W1, const void* b1, const void* W2,
                           medusa_dtype_t dt, int B, int d, int V, int K, int kmax,
                           int32_t* topk_ids, float* topk_vals, float* logits, void* ws,
                           int32_t* status, cudaStream_t stream, const TreeOut* tree) {
  const HeadsWs w = heads_ws_layout(B, d, V, K, kmax, dt);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  MergeTree mt{};
  if (dt == MEDUSA_F32) {
    float* y = reinterpret_cast<float*>(wsb);
    float* z = logits != nullptr ? logits : reinterpret_cast<float*>(wsb + w.y_bytes);
    int* seq_count = reinterpret_cast<int*>(wsb + w.y_bytes + w.part_bytes);
    if (tree != nullptr) mt = MergeTree{*tree, seq_count};
    launch(heads_f32_w1_kernel, dim3((d + 7) / 8, K), 256, 0, stream, static_cast<const float*>(h),
           static_cast<const float*>(W1), static_cast<const float*>(b1), B, d, K, y, seq_count);
    medusa_status_t st = check_launch("heads_f32_w1");
    if (st != MEDUSA_OK) return st;
    launch(heads_f32_w2_kernel, dim3((V + 7) / 8, K), 256, 0, stream, y,
           static_cast<const float*>(W2), B, d, V, K, z);
    st = check_launch("heads_f32_w2");
    if (st != MEDUSA_OK) return st;
    const MergeLayout lay{(long long)V, (long long)V, V, nullptr};
    launch(topk_merge_kernel, B * K * kMergeCtas, kMergeWarps * 32, 0, stream, z, nullptr, V, kmax,
           topk_ids, topk_vals, lay, mt);
    return check_launch("topk_merge");
  }

  __nv_bfloat16* Y = reinterpret_cast<__nv_bfloat16*>(wsb);
  float* part_vals = reinterpret_cast<float*>(wsb + w.y_bytes);
  int32_t* part_ids = reinterpret_cast<int32_t*>(wsb + w.y_bytes + w.part_bytes);

  CUtensorMap mA1, mB1, mA2, mB2;
  const int nb1 = round_nb(B);
  const int nb2 = round_nb(2 * B);
  if (!make_map_3d(&mA1, W1, d, d, K, kTileM) || !make_map_3d(&mB1, h, d, B, 1, nb1) ||
      !make_map_3d(&mA2, W2, d, V, K, kTileM) || !make_map_3d(&mB2, Y, d, 2 * B, K, nb2))
    return fail(MEDUSA_ERR_CUDA, "cuTensorMapEncodeTiled failed");

  GemmParams p1{};
  p1.rows_per_head = d;
  p1.n_heads = K;
  p1.d = d;
  p1.B = B;
  p1.tiles_per_head = (d + kTileM - 1) / kTileM;
  p1.n_tiles = p1.tiles_per_head * K;
  p1.b_head_stride = 0;
  p1.kmax = kmax;
  p1.h = static_cast<const __nv_bfloat16*>(h);
  p1.b1 = static_cast<const __nv_bfloat16*>(b1);
  p1.Y = Y;
  p1.status = status;
  p1.tile_counter = reinterpret_cast<int*>(wsb + w.y_bytes + 2 * w.part_bytes + w.sk_part_bytes +
                                           w.sk_flag_bytes);
  // Stream-K for the first GEMM when its few tiles would leave SMs idle for
  // part of the run: every CTA then takes the same number of k-blocks (at
  // least 8), and a tile cut between CTAs is finished by the one holding its
  // first k-block.
  {
    const int sms = num_sms();
    const int nkb = d / kTileK;
    const long long total_kb = (long long)p1.n_tiles * nkb;
    if (p1.n_tiles % sms != 0 && p1.n_tiles < 8 * sms && total_kb >= 8LL * sms) {
      p1.kpc = (int)((total_kb + sms - 1) / sms);
      p1.sk_grid = (int)((total_kb + p1.kpc - 1) / p1.kpc);
      p1.sk_part = reinterpret_cast<float*>(wsb + w.y_bytes + 2 * w.part_bytes);
      p1.sk_flag = reinterpret_cast<int*>(wsb + w.y_bytes + 2 * w.part_bytes + w.sk_part_bytes);
      launch(heads_flags_zero_kernel, 1, 256, 0, stream, p1.sk_flag, p1.sk_grid);
      const medusa_status_t zst = check_launch("heads stream-K flags");
      if (zst != MEDUSA_OK) return zst;
    }
  }
  medusa_status_t st = launch_gemm_nb<kModeW1>(nb1, mA1, mB1, p1, stream);
  if (st != MEDUSA_OK) return st;

  GemmParams p2 = p1;
  p2.kpc = 0;  // the second GEMM has many tiles per CTA: whole tiles, handed out dynamically
  p2.rows_per_head = V;
  p2.tiles_per_head = (V + kTileM - 1) / kTileM;
  p2.n_tiles = p2.tiles_per_head * K;
  p2.b_head_stride = 1;
  p2.logits = logits;
  p2.part_vals = part_vals;
  p2.part_ids = part_ids;
  // running lists when they fit: the merge then reads one list per CTA
  // instead of one per tile
  p2.run_lists = (K * B <= kRunMaxRows &&
                  gemm_alloc_bytes(nb2) + (size_t)K * B * kRunRowBytes <= (size_t)kSmemLimit)
                     ? 1
                     : 0;
  st = launch_gemm_nb<kModeW2>(nb2, mA2, mB2, p2, stream);
  if (st != MEDUSA_OK) return st;

  const long long C = (long long)(p2.run_lists ? gemm_grid(p2) : p2.tiles_per_head) * kmax;
  const MergeLayout lay{C, C, (int)C, nullptr};
  if (tree != nullptr) mt = MergeTree{*tree, p1.tile_counter + 1};
  launch(topk_merge_kernel, B * K * kMergeCtas, kMergeWarps * 32, 0, stream, part_vals, part_ids, C,
         kmax, topk_ids, topk_vals, lay, mt);
  return check_launch("topk_merge");
}

}  // namespace medusa
