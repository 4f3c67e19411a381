// Tree attention: every tree node attends to the cached prefix and to its
// own ancestors (and itself) in the tree.
//
// "Medusa Heads" glossary, "Attention arborescente et acceptation": all
// candidate tokens are appended to the input at once; a mask lets each one see
// only its ancestors, so one forward pass scores every branch.
//
// bf16 path (tcgen05): persistent, stream-K over balanced tiles.  A segment
// is 256 query rows of one (sequence, kv head) - the N nodes x G grouped query
// heads, as two M = 128 tiles - and its key tiles: ceil(P/128) prefix tiles,
// then the tree tiles (k_new/v_new, masked by the ancestor bitmask).  Every
// CTA takes an equal contiguous range of the concatenated tiles.  Roles:
//   warp 0      TMA producer: 128-key K and V tiles into a 2-stage ring, with
//               one word of tile facts per stage;
//   warp 1      MMA issuer: S = Q K^T into TMEM (one S/P buffer per M tile),
//               then O += P V with P as packed fp16 in TMEM (over the S
//               columns) and V as an M/N-major shared-memory operand;
//   warps 2,3   V converters: each landed V tile is rewritten in place from
//               bf16 to fp16; for the tree tiles of query group 0 they first
//               store the tree K/V into cache slots P + i;
//   warps 4..11 two softmax warpgroups, one query row per thread, holding a
//               whole 128-key tile of scores (warpgroup 0 gives up registers
//               to them): the row's scores come out of TMEM, max and sum stay
//               in the thread, O is rescaled in TMEM only when the row
//               maximum grows by more than 2^8 (the stale maximum cancels in
//               the final O / l).
// A piece that covers a whole segment writes its output rows directly.  Any
// other piece writes its normalised partial output and log2-sum-exp, then
// counts itself in a per-row counter; the row's last piece to arrive merges
// all of the row's partials (log-sum-exp weights) and writes the output row,
// so no separate merge pass follows the kernel.  The counters are zeroed by a
// small kernel before each launch.
//
// A V tile fp16 cannot carry flags its segment; an exact CUDA-core pass
// after the kernel recomputes the flagged segments' rows in fp32.
//
// fp32 path: one warp per query row on CUDA cores (small shapes).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "abi_internal.h"
#include "common.cuh"

namespace medusa {

constexpr int kAttnBN = 128;         // keys per tile (UMMA N of S = Q K^T)
constexpr int kAttnMT = 128;         // query rows per M tile (UMMA M)
constexpr int kAttnRows = 256;       // query rows per segment (two M tiles)
constexpr int kAttnStages = 2;       // K/V ring depth (64 KB per stage)
constexpr int kAttnThreads = 384;    // producer, MMA, two V converters, two softmax warpgroups
constexpr int kAttnRegsLow = 96;     // registers a thread in warpgroup 0
constexpr int kAttnRegsHigh = 200;   // registers a thread in the softmax warpgroups
constexpr float kRescaleLog2 = 8.f;  // lazy rescale threshold, log2 units
constexpr uint32_t kAttnTmemCols = 512;
constexpr int kAttnMaxB = 256;       // sequences per call (schedule table in shared memory)
constexpr int kAttnMinTiles = 4;     // smallest tile range a CTA takes

// 2^x with the SFU instruction (ex2.approx; relative error about 2^-22, -inf -> 0)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Register budget of a warpgroup (all four warps execute it together).  The
// shares must add up to no more than the registers the CTA was launched with
// (threads x registers per thread), or the increase waits for ever.
template <int N>
__device__ __forceinline__ void warpgroup_regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void warpgroup_regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// 5-D tiled load (no multicast), c0 innermost
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
      "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled store from shared memory (bulk-group completion), c0 innermost
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0,
                                             int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::
                   "l"(reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the shared-memory sources of every committed store have been read
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// every committed store has been performed
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// max of three (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// paired fp32 arithmetic (two lanes in one 64-bit register, sm_100)
__device__ __forceinline__ uint64_t f32x2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

struct AttnParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* Kc;
  __nv_bfloat16* Vc;
  const int32_t* prefix_len;
  const uint32_t* anc_mask;
  float* o_part;    // [n_seg, slots, DH / 4, 256] groups of 4 floats
  float* lse_part;  // [n_seg, slots, 256]
  unsigned int* row_count;  // [n_seg, 256] pieces of the row written so far (zeroed per call)
  // segments whose V has a tile fp16 cannot carry, recomputed by the exact
  // pass: a flag per segment, their count and list (zeroed per call)
  int* seg_flag;
  int* n_flag;
  int* flag_list;
  void* out;        // [B, N, Hq, DH], bf16 or fp32
  int out_f32;
  int B, N, Hq, Hkv, G, R, n_qg, T_tree, slots, cap, max_prefix, words, grid;
  int q_tma;  // Q tiles by bulk tensor loads (G divides 128)
  float scale_log2;
  int32_t* status;
};

template <int DH>
struct AttnSmem {
  static constexpr int kPanels = DH / 64;                  // 64-element (128 B) panels
  static constexpr int kQBytes = kAttnMT * DH * 2;         // one M tile of Q
  static constexpr int kKVBytes = kAttnBN * DH * 2;        // one K (or V) tile
  static constexpr int kPanelBytes = kAttnBN * 128;        // one 64-element panel of a tile
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + 2 * kQBytes;
  static constexpr int kVOff = kKOff + kAttnStages * kKVBytes;
  static constexpr int kBarOff = kVOff + kAttnStages * kKVBytes;
  // kv_full[S], kv_empty[S], v_ready[S], q_full[2], s_full[2], p_full[2], p_empty[2], drain,
  // copy_read[S]
  static constexpr int kNumBars = 4 * kAttnStages + 2 + 2 + 2 + 2 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kInfoOff = kMiscOff + 16;           // int info[kAttnStages]
  static constexpr int kAuxOff = kInfoOff + 16;  // int {bh, cache row0, segment, -}[kAttnStages]
  static constexpr int kCumOff = kAuxOff + 32;             // int cumT[kAttnMaxB + 1]
  static constexpr int kPrefOff = kCumOff + (kAttnMaxB + 1) * 4;  // int P[kAttnMaxB]
  static constexpr int kExitOff = (kPrefOff + kAttnMaxB * 4 + 7) & ~7;  // exit barrier
  static constexpr int kBytes = kExitOff + 8;
  static constexpr int kAlloc = kBytes + 1024;
};

// ----------------------------------------------------------------------------
// Schedule.  Segment = (sequence b, kv head, query group of 256 rows); its
// tiles are the ceil(P_b / 128) prefix tiles followed by the ceil(N / 128)
// tree tiles.  Segments are laid end to end (b-major) and every CTA takes an equal
// contiguous range of `per` tiles; a range cut at segment ends gives pieces,
// each written as one partial result (slot k = CTA - first CTA of the segment).
// ----------------------------------------------------------------------------
struct TileInfo {
  int b, kvh, qg, lt, tpre, ntiles, seg, slot, P, n_mt;
  bool first, last;
};

__device__ __forceinline__ void decode_tile(int t, const int* cumT, const int* pref,
                                            const AttnParams& p, int per, int t0, int t1,
                                            TileInfo& x) {
  int lo = 0, hi = p.B;  // cumT[lo] <= t < cumT[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cumT[mid] <= t) lo = mid;
    else hi = mid;
  }
  x.b = lo;
  x.P = pref[lo];
  x.tpre = (x.P + kAttnBN - 1) / kAttnBN;
  x.ntiles = x.tpre + p.T_tree;
  const int rem = t - cumT[lo];
  const int sib = rem / x.ntiles;
  x.lt = rem - sib * x.ntiles;
  x.kvh = sib / p.n_qg;
  x.qg = sib - x.kvh * p.n_qg;
  x.seg = (x.b * p.Hkv + x.kvh) * p.n_qg + x.qg;
  const int seg_start = t - x.lt;
  x.slot = (t0 / per) - seg_start / per;
  x.first = (t == t0) || (x.lt == 0);
  x.last = (t == t1 - 1) || (x.lt == x.ntiles - 1);
  x.n_mt = min(2, (p.R - x.qg * kAttnRows + kAttnMT - 1) / kAttnMT);
}

// Walks a CTA's tile range one tile at a time: decode_tile once, then only
// increments (the single-thread roles cannot afford a division per tile).
struct TileCursor {
  TileInfo x;
  int t, t0, t1, per, sib;
  const int* pref;
  const AttnParams* p;

  __device__ __forceinline__ void init(int t_, int t0_, int t1_, int per_, const int* cumT,
                                       const int* pref_, const AttnParams& pp) {
    t = t_;
    t0 = t0_;
    t1 = t1_;
    per = per_;
    pref = pref_;
    p = &pp;
    if (t < t1) {
      decode_tile(t, cumT, pref, pp, per, t0, t1, x);
      sib = x.kvh * pp.n_qg + x.qg;
    }
  }

  __device__ __forceinline__ void advance() {
    ++t;
    if (t >= t1) return;
    if (++x.lt == x.ntiles) {
      // next segment: next (kv head, query group) of this sequence, or the
      // next sequence
      x.lt = 0;
      if (++sib == p->Hkv * p->n_qg) {
        sib = 0;
        ++x.b;
        x.P = pref[x.b];
        x.tpre = (x.P + kAttnBN - 1) / kAttnBN;
        x.ntiles = x.tpre + p->T_tree;
      }
      x.kvh = sib / p->n_qg;
      x.qg = sib - x.kvh * p->n_qg;
      x.seg = (x.b * p->Hkv + x.kvh) * p->n_qg + x.qg;
      x.slot = t0 / per - t / per;
      x.n_mt = min(2, (p->R - x.qg * kAttnRows + kAttnMT - 1) / kAttnMT);
    }
    x.first = (x.lt == 0);
    x.last = (t == t1 - 1) || (x.lt == x.ntiles - 1);
  }
};

// What the MMA and converter warps need of a tile, packed into one word by the
// producer: bit 0 first tile of a piece (the accumulator starts over, a new Q
// tile is awaited), bit 1 both M tiles active, bit 2 last tile of a piece,
// bits 8..15 keys of the tile
// that are real (rows from there on are cleared in the converted V).
// Bit 16: a tree tile of query group 0, whose K/V the converter also stores
// into the caches (bit 17: the second tree tile, nodes 128..255).
__device__ __forceinline__ int pack_stage_info(const TileInfo& x) {
  const bool tree_tile = x.lt >= x.tpre;
  const int zero_from = tree_tile ? kAttnBN : min(kAttnBN, x.P - x.lt * kAttnBN);
  const bool copy = tree_tile && x.qg == 0;
  return (x.first ? 1 : 0) | (x.n_mt > 1 ? 2 : 0) | (x.last ? 4 : 0) | (zero_from << 8) |
         (copy ? 1 << 16 : 0) | (copy && x.lt > x.tpre ? 1 << 17 : 0);
}
__device__ __forceinline__ bool info_first(int w) { return (w & 1) != 0; }
__device__ __forceinline__ bool info_last(int w) { return (w & 4) != 0; }
__device__ __forceinline__ bool info_two(int w) { return (w & 2) != 0; }
__device__ __forceinline__ int info_zero_from(int w) { return (w >> 8) & 0xff; }
__device__ __forceinline__ bool info_copy(int w) { return (w & (1 << 16)) != 0; }
__device__ __forceinline__ bool info_second_tree(int w) { return (w & (1 << 17)) != 0; }

// cumT[b] = tiles of all segments of sequences < b; returns false if some
// prefix length is out of range.  Called by one full warp.
__device__ __forceinline__ bool build_schedule(const AttnParams& p, int* cumT, int* pref) {
  const int lane = threadIdx.x & 31;
  int run = 0;
  bool ok = true;
  if (lane == 0) cumT[0] = 0;
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int b = b0 + lane;
    int v = 0;
    if (b < p.B) {
      const int P = p.prefix_len[b];
      if (pref != nullptr) pref[b] = P;
      if (P < 0 || P > p.max_prefix || P + p.N > p.cap) ok = false;
      v = ((max(P, 0) + kAttnBN - 1) / kAttnBN + p.T_tree) * p.Hkv * p.n_qg;
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (b < p.B) cumT[b + 1] = run + v;
    run += __shfl_sync(0xffffffffu, v, 31);
  }
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ int tiles_per_cta(int total, int grid) {
  const int per = (total + grid - 1) / grid;
  return per < kAttnMinTiles ? kAttnMinTiles : per;
}

// 32 output values of query row r (within the segment's query rows) from
// column c0: row r is query head kvh * G + g of node r / G
struct OutRow {
  void* out;
  int out_f32, N, Hq, G;
};

template <int DH>
__device__ __forceinline__ void store_out_row32(const OutRow& q, int b, int kvh, int r, int c0,
                                                const float (&v)[32]) {
  const int node = r / q.G, g = r - node * q.G;
  const size_t base = (((size_t)b * q.N + node) * q.Hq + kvh * q.G + g) * DH + c0;
  if (q.out_f32) {
    float4* o = reinterpret_cast<float4*>(static_cast<float*>(q.out) + base);
#pragma unroll
    for (int c = 0; c < 8; ++c) o[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
  } else {
    uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(q.out) + base);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * c + 2 * q], v[8 * c + 2 * q + 1]);
        w[q] = *reinterpret_cast<const uint32_t*>(&b2);
      }
      o[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// The merge of a query row's pieces by the last one to arrive: weights
// 2^(lse_k - max lse), the partials (normalised O of each key range) summed
// with them and divided by the weights' sum.  The partials of other CTAs are
// read past L1 (they were released by a fence before their row count).
template <int DH>
__device__ __noinline__ void merge_row(const float* o_part, const float* lse_part, OutRow q,
                                       int b, int kvh, int r, size_t pbase, int row,
                                       unsigned int n_pieces) {
  constexpr int kFast = 4;  // pieces whose loads are all in flight together
  const float4* src0 = reinterpret_cast<const float4*>(o_part) + pbase * kAttnRows * (DH / 4) + row;
  const size_t piece_stride = (size_t)kAttnRows * (DH / 4);
  if (n_pieces <= kFast) {
    float lse[kFast];
#pragma unroll
    for (int k = 0; k < kFast; ++k)
      lse[k] = k < (int)n_pieces ? __ldcg(lse_part + (pbase + k) * kAttnRows + row) : -INFINITY;
    const float M = fmaxf(fmaxf(lse[0], lse[1]), fmaxf(lse[2], lse[3]));
    float w[kFast], wsum = 0.f;
#pragma unroll
    for (int k = 0; k < kFast; ++k) {
      w[k] = lse[k] == -INFINITY ? 0.f : exp2f(lse[k] - M);
      wsum += w[k];
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
    for (int k = 0; k < kFast; ++k) w[k] *= inv;
#pragma unroll 1
    for (int ch = 0; ch < DH / 32; ++ch) {
      float4 v[kFast][8];
#pragma unroll
      for (int k = 0; k < kFast; ++k)
#pragma unroll
        for (int c = 0; c < 8; ++c)
          v[k][c] = k < (int)n_pieces ? __ldcg(src0 + k * piece_stride + (ch * 8 + c) * kAttnRows)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
      float acc[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        acc[4 * c] = w[0] * v[0][c].x + w[1] * v[1][c].x + w[2] * v[2][c].x + w[3] * v[3][c].x;
        acc[4 * c + 1] = w[0] * v[0][c].y + w[1] * v[1][c].y + w[2] * v[2][c].y + w[3] * v[3][c].y;
        acc[4 * c + 2] = w[0] * v[0][c].z + w[1] * v[1][c].z + w[2] * v[2][c].z + w[3] * v[3][c].z;
        acc[4 * c + 3] = w[0] * v[0][c].w + w[1] * v[1][c].w + w[2] * v[2][c].w + w[3] * v[3][c].w;
      }
      store_out_row32<DH>(q, b, kvh, r, ch * 32, acc);
    }
    return;
  }
  float M = -INFINITY;
  for (unsigned int k = 0; k < n_pieces; ++k)
    M = fmaxf(M, __ldcg(lse_part + (pbase + k) * kAttnRows + row));
  float wsum = 0.f;
  for (unsigned int k = 0; k < n_pieces; ++k) {
    const float lse = __ldcg(lse_part + (pbase + k) * kAttnRows + row);
    wsum += lse == -INFINITY ? 0.f : exp2f(lse - M);
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll 1
  for (int ch = 0; ch < DH / 32; ++ch) {
    float acc[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c] = 0.f;
    for (unsigned int k = 0; k < n_pieces; ++k) {
      const float lse = __ldcg(lse_part + (pbase + k) * kAttnRows + row);
      const float w = lse == -INFINITY ? 0.f : exp2f(lse - M) * inv;
      const float4* src = src0 + k * piece_stride;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 v = __ldcg(src + (ch * 8 + c) * kAttnRows);
        acc[4 * c] += w * v.x;
        acc[4 * c + 1] += w * v.y;
        acc[4 * c + 2] += w * v.z;
        acc[4 * c + 3] += w * v.w;
      }
    }
    store_out_row32<DH>(q, b, kvh, r, ch * 32, acc);
  }
}

// Row counters of the in-kernel merge and the exact pass's segment flags and
// count, zeroed before every attention launch (one contiguous range).
__global__ void attn_zero_kernel(unsigned int* __restrict__ cnt, size_t n) {
  grid_dep_wait();
  grid_dep_launch();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    cnt[i] = 0u;
}

// The exact pass: every query row of every listed segment recomputed on CUDA
// cores from the bf16 inputs with fp32 arithmetic (one warp per row, lanes
// splitting dh, eight prefix keys per online-softmax update), overwriting the
// tensor-core kernel's output rows.  With no segment listed it only reads the
// count.
template <int DH>
__global__ void __launch_bounds__(256) tree_attn_exact_kernel(AttnParams p) {
  grid_dep_wait();
  grid_dep_launch();
  const int nf = *reinterpret_cast<volatile int*>(p.n_flag);
  if (nf == 0) return;
  constexpr int PER = DH / 32;
  const int lane = threadIdx.x & 31;
  const long long n_rows = (long long)nf * kAttnRows;
  const float scale = p.scale_log2 * 0.6931471805599453f;  // back to natural units
  for (long long e = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); e < n_rows;
       e += (long long)gridDim.x * 8) {
    const int seg = p.flag_list[e / kAttnRows];
    const int r = (seg % p.n_qg) * kAttnRows + static_cast<int>(e % kAttnRows);
    if (r >= p.R) continue;
    const int bh = seg / p.n_qg, b = bh / p.Hkv, kvh = bh - b * p.Hkv;
    const int node = r / p.G, g = r - node * p.G;
    const int P = p.prefix_len[b];
    float qv[PER], acc[PER];
    const __nv_bfloat16* qp = p.q + (((size_t)b * p.N + node) * p.Hq + kvh * p.G + g) * DH;
#pragma unroll
    for (int c = 0; c < PER; ++c) {
      qv[c] = __bfloat162float(qp[lane * PER + c]);
      acc[c] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    auto visit = [&](const __nv_bfloat16* kp, const __nv_bfloat16* vp) {
      float d = 0.f;
#pragma unroll
      for (int c = 0; c < PER; ++c) d += qv[c] * __bfloat162float(kp[lane * PER + c]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      const float sc = d * scale;
      const float mn = fmaxf(m, sc);
      const float corr = expf(m - mn), w = expf(sc - mn);
      l = l * corr + w;
#pragma unroll
      for (int c = 0; c < PER; ++c) acc[c] = acc[c] * corr + w * __bfloat162float(vp[lane * PER + c]);
      m = mn;
    };
    const size_t hb = ((size_t)b * p.Hkv + kvh) * p.cap;
    for (int t = 0; t < P; ++t) visit(p.Kc + (hb + t) * DH, p.Vc + (hb + t) * DH);
    for (int jn = 0; jn < p.N; ++jn) {
      if ((p.anc_mask[(size_t)node * p.words + (jn >> 5)] >> (jn & 31)) & 1u) {
        const size_t off = (((size_t)b * p.N + jn) * p.Hkv + kvh) * DH;
        visit(p.k_new + off, p.v_new + off);
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const size_t ob = (((size_t)b * p.N + node) * p.Hq + kvh * p.G + g) * DH;
    if (p.out_f32) {
#pragma unroll
      for (int c = 0; c < PER; ++c) static_cast<float*>(p.out)[ob + lane * PER + c] = acc[c] * inv;
    } else {
#pragma unroll
      for (int c = 0; c < PER; ++c)
        static_cast<__nv_bfloat16*>(p.out)[ob + lane * PER + c] = __float2bfloat16_rn(acc[c] * inv);
    }
  }
}

template <int DH>
__global__ void __launch_bounds__(kAttnThreads, 1)
    tree_attn_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmKn,
                        const __grid_constant__ CUtensorMap tmVn,
                        const __grid_constant__ CUtensorMap tmKs0,
                        const __grid_constant__ CUtensorMap tmVs0,
                        const __grid_constant__ CUtensorMap tmKs1,
                        const __grid_constant__ CUtensorMap tmVs1,
                        const __grid_constant__ CUtensorMap tmQ, AttnParams p) {
  // The launch before this one is always attn_zero_kernel, which waited for
  // every earlier grid: the inputs (q, k_new, v_new, the caches, prefix_len,
  // the mask) are final already.  Only the counters and flags that kernel
  // zeroes need its completion, so the wait for it (griddepcontrol.wait) is
  // taken by the threads that touch them, right before they do; the
  // schedule, the first loads and the first MMAs overlap the zeroing.
  grid_dep_launch();
  using L = AttnSmem<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  int* cumT = reinterpret_cast<int*>(smem + L::kCumOff);
  int* pref = reinterpret_cast<int*>(smem + L::kPrefOff);
  volatile int* sched_ok = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 8);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (warp == 0) {
    const bool ok = build_schedule(p, cumT, pref);
    if (lane == 0) *sched_ok = ok ? 1 : 0;
    __syncwarp();
  }
  __syncthreads();
  if (!*sched_ok) {
    if (threadIdx.x == 0 && blockIdx.x == 0) report(p.status, MEDUSA_ERR_DEVICE_CHECK);
    return;
  }
  const int total = cumT[p.B];
  const int per = tiles_per_cta(total, gridDim.x);
  const int t0 = blockIdx.x * per;
  const int t1 = min(t0 + per, total);
  if (t0 >= total) return;
  const int n = t1 - t0;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + kAttnStages;
  uint64_t* v_ready = bars + 2 * kAttnStages;  // V tile converted to fp16
  uint64_t* q_full = bars + 3 * kAttnStages;  // [m]
  uint64_t* s_full = q_full + 2;              // [m]
  uint64_t* p_full = s_full + 2;              // [m]
  uint64_t* p_empty = p_full + 2;             // [m]
  uint64_t* drain = p_empty + 2;
  // [stage] a tree tile's cache stores have read the stage (one barrier per
  // stage: the next copy from a stage needs every converter thread past this one)
  uint64_t* copy_read = drain + 1;
  uint64_t* exit_bar = reinterpret_cast<uint64_t*>(smem + L::kExitOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  int* stage_info = reinterpret_cast<int*>(smem + L::kInfoOff);
  int* stage_aux = reinterpret_cast<int*>(smem + L::kAuxOff);  // tree copy: bh, first cache row

  if (threadIdx.x == 0) {
    for (int i = 0; i < kAttnStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&v_ready[i], 64);
    }
    for (int m = 0; m < 2; ++m) {
      mbar_init(&q_full[m], p.q_tma ? 1 : 128);
      mbar_init(&s_full[m], 1);
      mbar_init(&p_full[m], 128);
      mbar_init(&p_empty[m], 1);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < kAttnStages; ++i) mbar_init(&copy_read[i], 1);
    mbar_init(exit_bar, kAttnThreads);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kAttnTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  // every warp reconverges first: lane 0 of some warps ran a role alone
  __syncwarp();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t tmem_o = tmem_base;           // O[m]: columns m*DH .. m*DH+DH-1
  const uint32_t tmem_s = tmem_base + 2 * DH;  // S[m] then P[m]: 128 columns each

  // Warpgroup 0 (producer, MMA issuer, V converters) needs few registers;
  // the softmax warpgroups 1 and 2 hold a whole 128-key tile of scores.
  // 128 x kAttnRegsLow + 256 x kAttnRegsHigh <= 384 x 168, the allocation of
  // the launch (the kernel is built at 168 registers a thread).
  static_assert(128 * kAttnRegsLow + 256 * kAttnRegsHigh <= kAttnThreads * 168,
                "register split exceeds the launch's allocation");
  if (warp < 4) {
  warpgroup_regs_dec<kAttnRegsLow>();
  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmKn);
      tma_prefetch_desc(&tmVn);
      const uint64_t pol = p.n_qg > 1 ? l2_policy_evict_last() : l2_policy_evict_first();
      TileCursor cur;
      cur.init(t0, t0, t1, per, cumT, pref, p);
      int j = 0;
      for (; j < n; ++j, cur.advance()) {
        const TileInfo& x = cur.x;
        const int st = j % kAttnStages;
        if (!mbar_wait_bounded(&kv_empty[st], ((j / kAttnStages) & 1) ^ 1u, abort_flag, p.status))
          break;
        // published with the stage (the kv_full arrive releases it): the
        // MMA and converter warps read it instead of walking the schedule
        const int bh = x.b * p.Hkv + x.kvh;
        stage_info[st] = pack_stage_info(x);
        stage_aux[4 * st] = bh;
        stage_aux[4 * st + 1] = x.P + (x.lt - x.tpre) * kAttnBN;
        stage_aux[4 * st + 2] = x.seg;
        mbar_arrive_expect_tx(&kv_full[st], 2 * L::kKVBytes);
        uint8_t* kdst = smem + L::kKOff + st * L::kKVBytes;
        uint8_t* vdst = smem + L::kVOff + st * L::kKVBytes;
#pragma unroll
        for (int pn = 0; pn < L::kPanels; ++pn) {
          if (x.lt < x.tpre) {
            const int key = x.lt * kAttnBN;
            tma_load_3d(kdst + pn * L::kPanelBytes, &tmK, &kv_full[st], pn * 64, key, bh, pol);
            tma_load_3d(vdst + pn * L::kPanelBytes, &tmV, &kv_full[st], pn * 64, key, bh, pol);
          } else {
            const int node = (x.lt - x.tpre) * kAttnBN;
            tma_load_4d(kdst + pn * L::kPanelBytes, &tmKn, &kv_full[st], pn * 64, x.kvh, node, x.b,
                        pol);
            tma_load_4d(vdst + pn * L::kPanelBytes, &tmVn, &kv_full[st], pn * 64, x.kvh, node, x.b,
                        pol);
          }
        }
      }
      const int first = j > kAttnStages ? j - kAttnStages : 0;
      for (int x = first; x < j; ++x) {
        int dummy_abort = 0;
        mbar_wait_bounded(&kv_full[x % kAttnStages], (x / kAttnStages) & 1, &dummy_abort, p.status);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // Order per tile j: PV(0,j), QK(0,j+1), PV(1,j), QK(1,j+1): each M tile
    // has one S/P buffer, and while one warpgroup computes its softmax the
    // tensor core works on the other M tile.  The loop is kept lean (one
    // thread, sharing its issue slots with two softmax warps): tile facts come
    // from the producer's stage info, the two M tiles are unrolled, and the
    // barrier phases are plain counters.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(kAttnMT, kAttnBN, 0);
      constexpr uint32_t idesc_pv = umma_idesc_f16(kAttnMT, DH, 1);
      // shared-memory descriptors built once; advancing a descriptor only adds
      // to its start-address field (16-byte units)
      const uint64_t dq0 = umma_desc_sw128(smem_u32(smem + L::kQOff));
      const uint64_t dk0 = umma_desc_sw128(smem_u32(smem + L::kKOff));
      const uint64_t dv0 = umma_desc_sw128_lbo(smem_u32(smem + L::kVOff), L::kPanelBytes, 1024);
      // S[m] = Q[m] K^T from stage st
      auto issue_qk = [&](int m, int st) {
        const uint64_t dq = dq0 + (uint64_t)((m * L::kQBytes) >> 4);
        const uint64_t dk = dk0 + (uint64_t)((st * L::kKVBytes) >> 4);
        const uint32_t d = tmem_s + m * kAttnBN;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          constexpr uint32_t qpanel = (kAttnMT * 128) >> 4, kpanel = L::kPanelBytes >> 4;
          const uint32_t qo = (kk >> 2) * qpanel + (kk & 3) * 2;
          const uint32_t ko = (kk >> 2) * kpanel + (kk & 3) * 2;
          umma_bf16(d, dq + qo, dk + ko, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[m]);
      };
      // O[m] (+)= P[m] V from stage st
      auto issue_pv = [&](int m, int st, uint32_t acc0) {
        const uint64_t dv = dv0 + (uint64_t)((st * L::kKVBytes) >> 4);
        const uint32_t d = tmem_o + m * DH;
        const uint32_t pcol = tmem_s + m * kAttnBN;
#pragma unroll
        for (int kk = 0; kk < kAttnBN / 16; ++kk) {
          // P in TMEM: 16 keys = 8 columns of packed fp16 pairs.
          // V (fp16 after conversion): M/N-major, 16 keys = two 8-row groups
          // of 1024 bytes; the second 64-element head-dimension panel sits
          // one tile-panel on.
          umma_bf16_ts(d, pcol + kk * 8, dv + (uint64_t)((kk * 16 * 128) >> 4), idesc_pv,
                       kk > 0 ? 1u : acc0);
        }
        umma_commit(&p_empty[m]);
      };
      uint32_t nq0 = 0, nq1 = 0, np0 = 0, np1 = 0;  // completed waits per barrier
      bool ok = mbar_wait_bounded(&kv_full[0], 0, abort_flag, p.status);
      int cur = ok ? stage_info[0] : 0;
      if (ok) ok = mbar_wait_bounded(&q_full[0], nq0++ & 1, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        if (info_two(cur)) {
          ok = mbar_wait_bounded(&q_full[1], nq1++ & 1, abort_flag, p.status);
          if (ok) {
            tc_fence_after();
            issue_qk(1, 0);
          }
        }
      }
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % kAttnStages;
        const int sn = (j + 1) % kAttnStages;
        const bool has_next = j + 1 < n;
        const bool two = info_two(cur);
        const uint32_t acc0 = info_first(cur) ? 0u : 1u;
        if (!mbar_wait_bounded(&v_ready[st], (j / kAttnStages) & 1, abort_flag, p.status) ||
            !mbar_wait_bounded(&p_full[0], np0++ & 1, abort_flag, p.status))
          break;
        tc_fence_after();
        issue_pv(0, st, acc0);
        if (!two) umma_commit(&kv_empty[st]);
        int nxt = 0;
        if (has_next) {
          if (!mbar_wait_bounded(&kv_full[sn], ((j + 1) / kAttnStages) & 1, abort_flag, p.status))
            break;
          nxt = stage_info[sn];
          if (info_first(nxt) &&
              !mbar_wait_bounded(&q_full[0], nq0++ & 1, abort_flag, p.status))
            break;
          tc_fence_after();
          issue_qk(0, sn);
        }
        if (two) {
          if (!mbar_wait_bounded(&p_full[1], np1++ & 1, abort_flag, p.status)) break;
          tc_fence_after();
          issue_pv(1, st, acc0);
          umma_commit(&kv_empty[st]);
        }
        if (has_next && info_two(nxt)) {
          if (info_first(nxt) &&
              !mbar_wait_bounded(&q_full[1], nq1++ & 1, abort_flag, p.status))
            break;
          tc_fence_after();
          issue_qk(1, sn);
        }
        cur = nxt;
      }
      umma_commit(drain);
      int dummy_abort = 0;
      mbar_wait_bounded(drain, 0, &dummy_abort, p.status);
    }
  } else {
    // ---------------- V converters (warps 2, 3) ----------------
    // Each landed V tile is rewritten in place from bf16 to fp16 (the value
    // product runs on fp16 P and V); rows past the prefix end of a partial
    // tile are cleared (their weights are zero, but 0 * NaN is not).  A tile
    // fp16 cannot carry - some |v| of 65536 or more, or all of a warp's |v|
    // below 2^-6, where fp16 loses mantissa bits - puts its segment on the
    // list of the exact pass that follows the kernel.  Inf or NaN in V is
    // reported as a device-check error.
    const int ct = (warp - 2) * 32 + lane;
    bool range_ok = true;
    uint32_t copy_par = 0;  // bit s: parity of the copies made from stage s
    for (int j = 0; j < n; ++j) {
      const int st = j % kAttnStages;
      if (!mbar_wait_bounded(&kv_full[st], (j / kAttnStages) & 1, abort_flag, p.status)) break;
      const int info = stage_info[st];
      const int zero_from = info_zero_from(info);
      uint4* vt = reinterpret_cast<uint4*>(smem + L::kVOff + st * L::kKVBytes);
      if (info_copy(info)) {
        // tree tile of query group 0: its K/V (still bf16) go to cache rows
        // P + node by bulk tensor stores, whose boxes hold exactly the
        // tile's real nodes; V is converted once the stores have read it
        if (ct == 0) {
          const bool second = info_second_tree(info);
          const CUtensorMap* mk = second ? &tmKs1 : &tmKs0;
          const CUtensorMap* mv = second ? &tmVs1 : &tmVs0;
          const int bh = stage_aux[4 * st], row0 = stage_aux[4 * st + 1];
          const uint8_t* ks = smem + L::kKOff + st * L::kKVBytes;
#pragma unroll
          for (int pn = 0; pn < L::kPanels; ++pn) {
            tma_store_3d(mk, ks + pn * L::kPanelBytes, pn * 64, row0, bh);
            tma_store_3d(mv, reinterpret_cast<const uint8_t*>(vt) + pn * L::kPanelBytes, pn * 64,
                         row0, bh);
          }
          bulk_commit_group();
          bulk_wait_read_all();
          mbar_arrive(&copy_read[st]);
        } else if (!mbar_wait_bounded(&copy_read[st], (copy_par >> st) & 1u, abort_flag,
                                      p.status)) {
          break;
        }
        copy_par ^= 1u << st;
      }
      constexpr int kChunks = L::kKVBytes / 16, kPanelChunks = L::kPanelBytes / 16;
      constexpr int kUnroll = 8;
      static_assert(kChunks % (64 * kUnroll) == 0, "V tile must split evenly over the converters");
      uint32_t vmax = 0u;  // largest |v| bit pattern seen (bf16 halves)
#pragma unroll 1
      for (int e0 = ct; e0 < kChunks; e0 += 64 * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) v[u] = vt[e0 + u * 64];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int row = ((e0 + u * 64) % kPanelChunks) >> 3;  // key within the tile
          uint32_t* w = &v[u].x;
          const bool keep = row < zero_from;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (keep) vmax = __vmaxu2(vmax, w[q] & 0x7FFF7FFFu);
            const __half2 h2 = __floats2half2_rn(__uint_as_float(w[q] << 16),
                                                 __uint_as_float(w[q] & 0xffff0000u));
            w[q] = keep ? *reinterpret_cast<const uint32_t*>(&h2) : 0u;
          }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) vt[e0 + u * 64] = v[u];
      }
      // 0x4780: the first bf16 past fp16's largest value 65504; 0x3C80: 2^-6;
      // 0x7F80 and above: inf or NaN
      const uint32_t vm = max(vmax & 0xffffu, vmax >> 16);
      if (vm >= 0x7F80u) range_ok = false;
      const uint32_t wmax = __reduce_max_sync(0xffffffffu, vm);
      if (lane == 0 && wmax < 0x7F80u && (wmax >= 0x4780u || (wmax != 0u && wmax < 0x3C80u))) {
        const int seg = stage_aux[4 * st + 2];
        grid_dep_wait();  // the flags are zeroed by the previous launch
        if (atomicCAS(&p.seg_flag[seg], 0, 1) == 0) p.flag_list[atomicAdd(p.n_flag, 1)] = seg;
      }
      fence_proxy_async_smem();
      mbar_arrive(&v_ready[st]);
    }
    if (ct == 0) bulk_wait_all();
    if (!range_ok) report(p.status, MEDUSA_ERR_DEVICE_CHECK);
  }
  } else {
    warpgroup_regs_inc<kAttnRegsHigh>();
    // ---------------- softmax warpgroups (M tile 0: warps 4-7, 1: 8-11) ----------------
    const int m = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int rl = quad * 32 + lane;  // row within the M tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t srow = tmem_s + lane_off + m * kAttnBN;
    uint8_t* qtile = smem + L::kQOff + m * L::kQBytes;

    // Q rows of a segment into the swizzled K-major tile (zeros past R).
    // When G divides 128 the tile is one box of the query tensor seen as
    // [B][N][Hkv][G][DH] (rows = node-major (node, g) pairs, nodes past N
    // zero-filled), fetched by one bulk tensor load per 64-column panel.
    auto load_q = [&](const TileInfo& x) {
      if (p.q_tma) {
        if (rl == 0) {
          const int node0 = (x.qg * kAttnRows + m * kAttnMT) / p.G;
          mbar_arrive_expect_tx(&q_full[m], L::kQBytes);
#pragma unroll
          for (int pn = 0; pn < L::kPanels; ++pn)
            tma_load_5d(qtile + pn * (kAttnMT * 128), &tmQ, &q_full[m], pn * 64, 0, x.kvh, node0,
                        x.b);
        }
        return;
      }
      const int r = x.qg * kAttnRows + m * kAttnMT + rl;
      const bool valid = r < p.R;
      const int node = valid ? r / p.G : 0;
      const int g = valid ? r - node * p.G : 0;
      const uint4* qsrc = reinterpret_cast<const uint4*>(
          p.q + (((size_t)x.b * p.N + node) * p.Hq + x.kvh * p.G + g) * DH);
#pragma unroll
      for (int c = 0; c < DH / 8; ++c) {
        const uint4 v = valid ? qsrc[c] : make_uint4(0u, 0u, 0u, 0u);
        const int pn = c >> 3, cc = c & 7;
        *reinterpret_cast<uint4*>(qtile + pn * (kAttnMT * 128) + rl * 128 + ((cc ^ (rl & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      mbar_arrive(&q_full[m]);
    };

    int tcount = 0;
    bool q_ready = false;
    bool ok = true;
    float m_used = -INFINITY, l_run = 0.f;
    uint32_t mw[8];
    int jj = 0;
    int piece_lt0 = 0;  // the segment tile the current piece starts at
    const OutRow out_row{p.out, p.out_f32, p.N, p.Hq, p.G};
    TileCursor cur;
    cur.init(t0, t0, t1, per, cumT, pref, p);
    for (int j = 0; ok && j < n; ++j, cur.advance()) {
      const TileInfo x = cur.x;
      if (m >= x.n_mt) continue;
      const int r = x.qg * kAttnRows + m * kAttnMT + rl;
      const bool valid = r < p.R;
      if (x.first) {
        if (!q_ready) load_q(x);
        q_ready = false;
        const int node = valid ? r / p.G : 0;
#pragma unroll
        for (int w = 0; w < 8; ++w)
          mw[w] = (valid && w < p.words) ? p.anc_mask[(size_t)node * p.words + w] : 0xffffffffu;
        m_used = -INFINITY;
        l_run = 0.f;
        jj = 0;
        piece_lt0 = x.lt;
      }
      if (!mbar_wait_bounded(&s_full[m], tcount & 1, abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (x.last && j + 1 < n) {
        // every QK of this piece is done: load the next piece's Q now, so the
        // MMA warp can run ahead into it
        TileCursor nx = cur;
        nx.advance();
        if (m < nx.x.n_mt) {
          load_q(nx.x);
          q_ready = true;
        }
      }
      const bool tree_tile = x.lt >= x.tpre;
      const int kbase = tree_tile ? (x.lt - x.tpre) * kAttnBN : x.lt * kAttnBN;
      const int key_end = tree_tile ? p.N : x.P;
      const bool full_tile = !tree_tile && kbase + kAttnBN <= key_end;
      // the tile's four mask words, picked without dynamic register indexing
      uint32_t tw[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      if (tree_tile) {
        const bool upper = x.lt > x.tpre;  // second tree tile: nodes 128..255
#pragma unroll
        for (int q = 0; q < 4; ++q) tw[q] = upper ? mw[4 + q] : mw[q];
      }
      // One pass over the whole tile: all 128 scores of the row come out of
      // TMEM with one wait.  The exponent base is the running maximum m_used
      // (log2 units); a tile whose maximum exceeds it by more than 2^8 (or the
      // first tile of a piece) moves the base and rescales O and l, so that
      // every stored weight stays <= 2^8 (well inside fp16).
      float sv[kAttnBN];
      {
        uint32_t r[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32_raw(srow + q * 32, r[q]);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          tmem_regs_after_wait(r[q]);
#pragma unroll
          for (int c = 0; c < 32; ++c) sv[q * 32 + c] = __uint_as_float(r[q][c]);
        }
      }
      if (!full_tile) {
        // visible keys, 32 at a time: below the key end and set in the
        // ancestor bitmask (the words are selected, not indexed, so the mask
        // stays in registers)
        const int nv = min(max(key_end - kbase, 0), kAttnBN);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int nq = min(max(nv - q * 32, 0), 32);
          const uint32_t vis = (nq >= 32 ? 0xffffffffu : ((1u << nq) - 1u)) & tw[q];
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (!((vis >> c) & 1u)) sv[q * 32 + c] = -INFINITY;
        }
      }
      // row maximum: three-input max in four independent chains
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < kAttnBN; c += 2)
        m4[(c >> 1) & 3] = fmax3(m4[(c >> 1) & 3], sv[c], sv[c + 1]);
      const float mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * p.scale_log2;
      const bool need = (m_used == -INFINITY) ? (mx != -INFINITY) : (mx > m_used + kRescaleLog2);
      if (__any_sync(0xffffffffu, need)) {
        const float new_m = need ? mx : m_used;
        const float corr = (need && m_used != -INFINITY) ? ex2_approx(m_used - new_m) : 1.f;
        if (jj > 0) {
          // O holds earlier tiles (their PV is done: this tile's QK was
          // issued after it)
#pragma unroll 1
          for (int ch = 0; ch < DH / 32; ++ch) {
            float o[32];
            const uint32_t ta = tmem_o + lane_off + m * DH + ch * 32;
            tmem_ld32(ta, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= corr;
            tmem_st32(ta, o);
          }
        }
        l_run *= corr;
        m_used = new_m;
      }
      // weights 2^(s * scale - m) on key pairs: the exponent argument and the
      // running sums use the paired fp32 instructions; four partial sums.  P
      // (packed fp16 pairs, 64 columns) overwrites the first half of S, which
      // is already in registers.
      const float nbase = m_used == -INFINITY ? 0.f : -m_used;
      const uint64_t scale2 = f32x2_pack(p.scale_log2, p.scale_log2);
      const uint64_t nbase2 = f32x2_pack(nbase, nbase);
      uint64_t part[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = hq * 64 + 2 * e;
          float x0, x1;
          f32x2_unpack(f32x2_fma(f32x2_pack(sv[c], sv[c + 1]), scale2, nbase2), x0, x1);
          const float a0 = ex2_approx(x0);
          const float a1 = ex2_approx(x1);
          part[e & 3] = f32x2_add(part[e & 3], f32x2_pack(a0, a1));
          const __half2 h2 = __floats2half2_rn(a0, a1);
          pk[e] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        tmem_st32_u(srow + hq * 32, pk);
      }
      {
        float s0, s1;
        f32x2_unpack(f32x2_add(f32x2_add(part[0], part[1]), f32x2_add(part[2], part[3])), s0, s1);
        l_run += s0 + s1;
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[m]);
      if (x.last) {
        // the piece's results go to memory the previous launch zeroes (row
        // counters) or that follows it in the stream order
        grid_dep_wait();
        // the piece ends: wait for its last PV
        if (!mbar_wait_bounded(&p_empty[m], tcount & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        if (piece_lt0 == 0 && x.lt == x.ntiles - 1) {
          // the piece is the whole segment: O / l is the row's output
#pragma unroll 1
          for (int ch = 0; ch < DH / 32; ++ch) {
            float o[32];
            tmem_ld32(tmem_o + lane_off + m * DH + ch * 32, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= inv;
            if (valid) store_out_row32<DH>(out_row, x.b, x.kvh, r, ch * 32, o);
          }
        } else {
          // a normalised partial O and its log2-sum-exp; the row's last piece
          // to arrive (counted per row) merges all of them
          const size_t pbase = (size_t)x.seg * p.slots;
          const size_t piece = pbase + x.slot;
          // column-group-major partial: a warp's 32 rows of one group of 4
          // columns are 512 contiguous bytes
          float4* dst = reinterpret_cast<float4*>(p.o_part) + piece * kAttnRows * (DH / 4) +
                        m * kAttnMT + rl;
#pragma unroll 1
          for (int ch = 0; ch < DH / 32; ++ch) {
            float o[32];
            tmem_ld32(tmem_o + lane_off + m * DH + ch * 32, o);
            if (valid) {
#pragma unroll
              for (int c = 0; c < 8; ++c)
                dst[(ch * 8 + c) * kAttnRows] = make_float4(o[4 * c] * inv, o[4 * c + 1] * inv,
                                                            o[4 * c + 2] * inv, o[4 * c + 3] * inv);
            }
          }
          if (valid) {
            const int row = m * kAttnMT + rl;
            p.lse_part[piece * kAttnRows + row] = l_run > 0.f ? m_used + log2f(l_run) : -INFINITY;
            const int seg_t0 = t0 + j - x.lt;  // the segment's first tile (global index)
            const unsigned int n_pieces =
                static_cast<unsigned int>((seg_t0 + x.ntiles - 1) / per - seg_t0 / per + 1);
            // release this piece, count it; the counter wraps to 0 at the last
            __threadfence();
            const unsigned int before =
                atomicInc(&p.row_count[(size_t)x.seg * kAttnRows + row], n_pieces - 1);
            if (before == n_pieces - 1) {
              __threadfence();
              merge_row<DH>(p.o_part, p.lse_part, out_row, x.b, x.kvh, r, pbase, row, n_pieces);
            }
          }
        }
        tc_fence_before();
      }
      ++tcount;
      ++jj;
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
    tmem_dealloc(tmem_base, kAttnTmemCols);
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
  grid_dep_wait();
  grid_dep_launch();
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
  grid_dep_wait();
  grid_dep_launch();
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
  // the cached prefix eight keys at a time: their loads are in flight
  // together, then one online-softmax update takes all eight
  constexpr int KB = 8;
  int t = 0;
  for (; t + KB <= P; t += KB) {
    float sc[KB];
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      const float* kp = Kc + (hb + t + u) * dh;
      float sd = 0.f;
#pragma unroll
      for (int e = 0; e < MAXPER; ++e)
        if (e < per) sd += qv[e] * kp[lane * per + e];
      sc[u] = sd;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int u = 0; u < KB; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
    }
    float mn = m;
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      sc[u] *= scale;
      mn = fmaxf(mn, sc[u]);
    }
    const float corr = expf(m - mn);
    l *= corr;
#pragma unroll
    for (int e = 0; e < MAXPER; ++e) acc[e] *= corr;
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      const float pw = expf(sc[u] - mn);
      const float* vp = Vc + (hb + t + u) * dh;
      l += pw;
#pragma unroll
      for (int e = 0; e < MAXPER; ++e)
        if (e < per) acc[e] += pw * vp[lane * per + e];
    }
    m = mn;
  }
  for (; t < P; ++t) visit(Kc + (hb + t) * dh, Vc + (hb + t) * dh);
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

struct Plan {
  int n_qg, T_tree, slots;
};

Plan plan(int N, int Hq, int Hkv, int max_prefix) {
  Plan pl{};
  const int R = N * (Hq / Hkv);
  pl.n_qg = (R + kAttnRows - 1) / kAttnRows;
  pl.T_tree = (N + kAttnBN - 1) / kAttnBN;
  const int max_seg_tiles = (max_prefix + kAttnBN - 1) / kAttnBN + pl.T_tree;
  // the pieces a segment can be cut into
  pl.slots = (max_seg_tiles + kAttnMinTiles - 1) / kAttnMinTiles + 1;
  return pl;
}

}  // namespace

size_t tree_attention_workspace_size(int B, int N, int Hq, int Hkv, int dh, int max_prefix,
                                     medusa_dtype_t dt) {
  if (dt == MEDUSA_F32) return 0;
  const Plan pl = plan(N, Hq, Hkv, max_prefix);
  const size_t n_seg = (size_t)B * Hkv * pl.n_qg;
  const size_t seg_rows = n_seg * kAttnRows;
  const size_t rows = seg_rows * pl.slots;
  // partials, log-sum-exps, then one zeroed range: row counters, segment
  // flags, the flag count; then the flagged-segment list
  return align256(rows * dh * 4) + align256(rows * 4) + align256((seg_rows + n_seg + 1) * 4) +
         align256(n_seg * 4);
}

template <int DH>
static medusa_status_t launch_bf16(AttnParams& p, void* out, int out_f32, cudaStream_t stream) {
  using L = AttnSmem<DH>;
  // caches [B*Hkv][cap][DH]; tree K/V [B][N][Hkv][DH]; boxes of 128 keys x 64
  // head dims (one 128-byte swizzled panel)
  CUtensorMap mK, mV, mKn, mVn;
  const uint64_t dc[3] = {DH, (uint64_t)p.cap, (uint64_t)p.B * p.Hkv};
  const uint64_t sc[2] = {DH * 2, (uint64_t)p.cap * DH * 2};
  const uint32_t bc[3] = {64, kAttnBN, 1};  // 64 head dims x 128 keys
  const uint64_t dn[4] = {DH, (uint64_t)p.Hkv, (uint64_t)p.N, (uint64_t)p.B};
  const uint64_t sn[3] = {DH * 2, (uint64_t)p.Hkv * DH * 2, (uint64_t)p.N * p.Hkv * DH * 2};
  const uint32_t bn[4] = {64, 1, kAttnBN, 1};
  // tree K/V stores into the caches: boxes of exactly the real nodes of the
  // first and (N > 128) second tree tile
  CUtensorMap mKs0, mVs0, mKs1, mVs1;
  const uint32_t bs0[3] = {64, (uint32_t)(p.N < kAttnBN ? p.N : kAttnBN), 1};
  const uint32_t bs1[3] = {64, (uint32_t)(p.N > kAttnBN ? p.N - kAttnBN : 1), 1};
  // queries as [B][N][Hkv][G][DH]: a box of 64 columns x G heads x 128 / G nodes
  CUtensorMap mQ;
  p.q_tma = (kAttnMT % p.G == 0) ? 1 : 0;
  const uint64_t dq[5] = {DH, (uint64_t)p.G, (uint64_t)p.Hkv, (uint64_t)p.N, (uint64_t)p.B};
  const uint64_t sq[4] = {DH * 2, (uint64_t)p.G * DH * 2, (uint64_t)p.Hq * DH * 2,
                          (uint64_t)p.N * p.Hq * DH * 2};
  const uint32_t bq[5] = {64, (uint32_t)(p.q_tma ? p.G : 1), 1,
                          (uint32_t)(p.q_tma ? kAttnMT / p.G : 1), 1};
  if (!make_tmap_bf16(&mQ, p.q, 5, dq, sq, bq))
    return fail(MEDUSA_ERR_CUDA, "tree_attention: cuTensorMapEncodeTiled failed");
  if (!make_tmap_bf16(&mK, p.Kc, 3, dc, sc, bc) || !make_tmap_bf16(&mV, p.Vc, 3, dc, sc, bc) ||
      !make_tmap_bf16(&mKn, p.k_new, 4, dn, sn, bn) ||
      !make_tmap_bf16(&mVn, p.v_new, 4, dn, sn, bn) ||
      !make_tmap_bf16(&mKs0, p.Kc, 3, dc, sc, bs0) || !make_tmap_bf16(&mVs0, p.Vc, 3, dc, sc, bs0) ||
      !make_tmap_bf16(&mKs1, p.Kc, 3, dc, sc, bs1) || !make_tmap_bf16(&mVs1, p.Vc, 3, dc, sc, bs1))
    return fail(MEDUSA_ERR_CUDA, "tree_attention: cuTensorMapEncodeTiled failed");
  if (cudaFuncSetAttribute(tree_attn_tc_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           L::kAlloc) != cudaSuccess)
    return fail(MEDUSA_ERR_CUDA, "cudaFuncSetAttribute(tree_attention) failed");
  // the warpgroups' register shares must fit in what the launch allocates,
  // or the softmax warpgroups' increase would wait for ever: checked against
  // the registers the kernel was built with
  {
    static int regs = 0;
    if (regs == 0) {
      cudaFuncAttributes fa{};
      if (cudaFuncGetAttributes(&fa, tree_attn_tc_kernel<DH>) != cudaSuccess)
        return fail(MEDUSA_ERR_CUDA, "cudaFuncGetAttributes(tree_attention) failed");
      regs = fa.numRegs;
    }
    if (128 * kAttnRegsLow + 256 * kAttnRegsHigh > kAttnThreads * regs)
      return fail(MEDUSA_ERR_UNSUPPORTED, "tree_attention: register split exceeds the build's");
  }
  p.grid = device_sm_count();  // persistent: one CTA per SM
  p.out = out;
  p.out_f32 = out_f32;
  const size_t n_count = (size_t)p.B * p.Hkv * p.n_qg * (kAttnRows + 1) + 1;
  launch(attn_zero_kernel, (int)((n_count + 255) / 256 < 1024 ? (n_count + 255) / 256 : 1024), 256,
         0, stream, p.row_count, n_count);
  medusa_status_t st = check_launch("tree_attention_counters");
  if (st != MEDUSA_OK) return st;
  launch(tree_attn_tc_kernel<DH>, p.grid, kAttnThreads, L::kAlloc, stream, mK, mV, mKn, mVn, mKs0,
         mVs0, mKs1, mVs1, mQ, p);
  st = check_launch("tree_attention");
  if (st != MEDUSA_OK) return st;
  launch(tree_attn_exact_kernel<DH>, p.grid, 256, 0, stream, p);
  return check_launch("tree_attention_exact");
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
    launch(tree_kv_write_f32_kernel, blocks, 256, 0, stream, static_cast<const float*>(k_new),
           static_cast<const float*>(v_new), static_cast<float*>(Kc), static_cast<float*>(Vc),
           prefix_len, B, N, Hkv, dh, cap, max_prefix, status);
    medusa_status_t st = check_launch("tree_kv_write_f32");
    if (st != MEDUSA_OK) return st;
    const int rows = B * N * Hq;
    launch(tree_attn_f32_kernel, (rows + 7) / 8, 256, 0, stream, static_cast<const float*>(q),
           static_cast<const float*>(k_new), static_cast<const float*>(v_new),
           static_cast<const float*>(Kc), static_cast<const float*>(Vc), prefix_len, anc_mask, B, N,
           Hq, Hkv, dh, cap, max_prefix, words, scale, out, out_f32);
    return check_launch("tree_attention_f32");
  }
  const Plan pl = plan(N, Hq, Hkv, max_prefix);
  AttnParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.Kc = static_cast<__nv_bfloat16*>(Kc);
  p.Vc = static_cast<__nv_bfloat16*>(Vc);
  p.prefix_len = prefix_len;
  p.anc_mask = anc_mask;
  const size_t n_seg = (size_t)B * Hkv * pl.n_qg;
  const size_t seg_rows = n_seg * kAttnRows;
  const size_t rows = seg_rows * pl.slots;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  p.o_part = reinterpret_cast<float*>(w8);
  p.lse_part = reinterpret_cast<float*>(w8 + align256(rows * dh * 4));
  p.row_count = reinterpret_cast<unsigned int*>(w8 + align256(rows * dh * 4) + align256(rows * 4));
  p.seg_flag = reinterpret_cast<int*>(p.row_count + seg_rows);
  p.n_flag = p.seg_flag + n_seg;
  p.flag_list = reinterpret_cast<int*>(w8 + align256(rows * dh * 4) + align256(rows * 4) +
                                       align256((seg_rows + n_seg + 1) * 4));
  p.B = B;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.R = N * p.G;
  p.n_qg = pl.n_qg;
  p.T_tree = pl.T_tree;
  p.slots = pl.slots;
  p.cap = cap;
  p.max_prefix = max_prefix;
  p.words = words;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = status;
  if (dh == 128) return launch_bf16<128>(p, out, out_f32, stream);
  return launch_bf16<64>(p, out, out_f32, stream);
}

}  // namespace medusa
