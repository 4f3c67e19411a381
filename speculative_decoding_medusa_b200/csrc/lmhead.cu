// Verification straight from the tree nodes' hidden states.
//
// "Medusa Heads" glossary, "Attention arborescente et acceptation": one
// forward pass scores every candidate of the tree, and the longest branch the
// base model agrees with is kept; the base model's scores at a node are its
// lm_head applied to the node's last hidden state.  Materialising those
// verify logits ([B*N, V] fp32 or bf16) only to reduce each row to an argmax
// (greedy) or to a log-sum-exp and an entropy (typical) costs a write and a
// read of B*N*V values; here the lm_head GEMM reduces its own tiles.
//
// One tcgen05 GEMM, D[v, c] = lm_head[v, :] . hidden[c, :], with vocabulary
// rows in the MMA's M (128 per tile) and the B*N node columns in N: a column
// block of up to 512 columns is two N <= 256 MMAs per 16-deep step into the
// two halves of a 512-column TMEM accumulator, so each lm_head tile is read
// from HBM once per column block.  Roles (192 threads):
//   warp 0     TMA producer: a 128 x 64 lm_head tile and the block's two
//              256 x 64 hidden tiles per stage;
//   warp 1     MMA issuer (and TMEM owner);
//   warps 2-5  epilogue: per 32-column group a transposing butterfly over the
//              32 rows of each warp leaves lane c holding column c's maximum
//              (lowest index on ties) and, for typical acceptance, its
//              sums exp(z/T - max/T) and exp(..) z/T; the four warps' results
//              merge through shared memory into the CTA's running per-column
//              record, written out once per column block.
// A CTA takes a contiguous range of (column block, vocabulary tile) units;
// each column's records from the CTAs that covered it are merged by the path
// kernel of the verification, which then runs the usual acceptance.  The
// epilogue releases each TMEM half as soon as it has read it, so the next
// tile's first MMAs into half 0 overlap the reduction of half 1.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "abi_internal.h"
#include "common.cuh"

namespace medusa {

constexpr int kLmTileM = 128;    // vocabulary rows per tile (UMMA M)
constexpr int kLmTileK = 64;     // bf16 per 128-byte swizzled row
constexpr int kLmHalf = 256;     // columns per MMA (UMMA N <= 256)
constexpr int kLmBlock = 512;    // columns per block (two halves)
constexpr int kLmStages = 4;    // a stage: one k-block of lm_head and of one hidden half
constexpr int kLmThreads = 192;

struct LmParams {
  int V, d, C;                  // vocabulary, reduction length, columns (B * N)
  int n_vt, n_cb, n_units, per;  // tiles, column blocks, units, units per CTA
  int n_slots;                  // records per column
  int typical;
  float inv_T;
  float t_log2;                 // log2(e) / T: exp(x / T) = 2^(x * t_log2)
  float* logits;                // [C, V] fp32, or null
  RowPart* part;                // [C, n_slots]
  int32_t* status;
};

struct LmSmem {
  static constexpr int kABytes = kLmTileM * kLmTileK * 2;  // 16 KB
  static constexpr int kBHalfBytes = kLmHalf * kLmTileK * 2;  // 32 KB
  static constexpr int kBBytes = kBHalfBytes;
  static constexpr int kAOff = 0;
  static constexpr int kBOff = kAOff + kLmStages * kABytes;
  static constexpr int kRedOff = kBOff + kLmStages * kBBytes;   // RowPart red[4][256]
  static constexpr int kScrOff = kRedOff + 4 * kLmHalf * 16;    // float [4][32][33]
  static constexpr int kBarOff = kScrOff + 4 * 32 * 33 * 4;
  // full[S], empty[S], tfull, tempty[2], drain, epi, exit
  static constexpr int kNumBars = 2 * kLmStages + 6;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

// columns of block cb, and the N of its two MMAs (0: half unused)
__device__ __forceinline__ void block_shape(const LmParams& p, int cb, int& ncols, int& nb0,
                                            int& nb1) {
  ncols = min(kLmBlock, p.C - cb * kLmBlock);
  const int padded = round16(ncols);
  nb0 = min(kLmHalf, padded);
  nb1 = padded > kLmHalf ? padded - kLmHalf : 0;
}

// 2^x with the SFU instruction (relative error about 2^-22; -inf -> 0)
__device__ __forceinline__ float lm_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// merge record b into a (same column); s and t are relative to exp(maxz/T)
__device__ __forceinline__ void merge_record(RowPart& a, const RowPart& b, bool typical,
                                             float t_log2) {
  if (typical) {
    const float M = fmaxf(a.maxz, b.maxz);
    const float wa = a.maxz == -INFINITY ? 0.f : lm_ex2((a.maxz - M) * t_log2);
    const float wb = b.maxz == -INFINITY ? 0.f : lm_ex2((b.maxz - M) * t_log2);
    a.s = a.s * wa + b.s * wb;
    a.t = a.t * wa + b.t * wb;
  }
  if (better(b.maxz, b.idx, a.maxz, a.idx)) {
    a.maxz = b.maxz;
    a.idx = b.idx;
  }
}

__device__ __forceinline__ RowPart empty_record() {
  RowPart r;
  r.maxz = -INFINITY;
  r.idx = 0x7fffffff;
  r.s = 0.f;
  r.t = 0.f;
  return r;
}


// Transposing butterfly over the 32 rows of a warp for 32 columns at once:
// lane l starts with its row's values for columns 0..31; after five rounds
// (16 + 8 + 4 + 2 + 1 exchanges) v[0], id[0] hold column l's best value of
// the 32 rows and its lowest index.
__device__ __forceinline__ void warp_colmax32(float (&v)[32], int (&id)[32], int lane) {
#pragma unroll
  for (int h = 16; h > 0; h >>= 1) {
    const bool upper = (lane & h) != 0;  // keeps columns j + h of those still held
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const float sv = upper ? v[j] : v[j + h];
      const int si = upper ? id[j] : id[j + h];
      const float kv = upper ? v[j + h] : v[j];
      const int ki = upper ? id[j + h] : id[j];
      const float rv = __shfl_xor_sync(0xffffffffu, sv, h);
      const int ri = __shfl_xor_sync(0xffffffffu, si, h);
      const bool take = better(rv, ri, kv, ki);
      v[j] = take ? rv : kv;
      id[j] = take ? ri : ki;
    }
  }
}

// the same butterfly for two sums per column: a[0], b[0] end as column l's
__device__ __forceinline__ void warp_colsum32x2(float (&a)[32], float (&b)[32], int lane) {
#pragma unroll
  for (int h = 16; h > 0; h >>= 1) {
    const bool upper = (lane & h) != 0;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const float sa = upper ? a[j] : a[j + h];
      const float sb = upper ? b[j] : b[j + h];
      const float ka = upper ? a[j + h] : a[j];
      const float kb = upper ? b[j + h] : b[j];
      a[j] = ka + __shfl_xor_sync(0xffffffffu, sa, h);
      b[j] = kb + __shfl_xor_sync(0xffffffffu, sb, h);
    }
  }
}

__global__ void __launch_bounds__(kLmThreads, 1)
    lmhead_reduce_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB, LmParams p) {
  grid_dep_wait();
  grid_dep_launch();
  using L = LmSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = bars + kLmStages;
  uint64_t* tfull = bars + 2 * kLmStages;
  uint64_t* tempty = tfull + 1;  // [half]
  uint64_t* drain = tfull + 3;
  uint64_t* epi = tfull + 4;
  uint64_t* exit_bar = tfull + 5;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nkb = p.d / kLmTileK;
  const int u0 = blockIdx.x * p.per;
  const int u1 = min(u0 + p.per, p.n_units);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(&tempty[0], 128);
    mbar_init(&tempty[1], 128);
    mbar_init(drain, 1);
    mbar_init(epi, 128);
    mbar_init(exit_bar, kLmThreads);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 2 * kLmHalf);
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
      const uint64_t pol_a = l2_policy_evict_first();  // lm_head: read once
      const uint64_t pol_b = l2_policy_evict_last();   // hidden: read by every tile
      int g = 0;
      bool ok = true;
      for (int u = u0; ok && u < u1; ++u) {
        const int cb = u / p.n_vt, vt = u - cb * p.n_vt;
        int ncols, nb0, nb1;
        block_shape(p, cb, ncols, nb0, nb1);
        // stages in order (kb, half): the second half's copy of the lm_head
        // k-block comes from L2
        const int nh = nb1 > 0 ? 2 : 1;
        for (int st = 0; st < nkb * nh; ++st, ++g) {
          const int kb = st / nh, h = st - kb * nh;
          const int s = g % kLmStages;
          if (!mbar_wait_bounded(&empty[s], ((g / kLmStages) & 1) ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], L::kABytes + L::kBBytes);
          tma_load_3d(smem + L::kAOff + s * L::kABytes, &tmA, &full[s], kb * kLmTileK,
                      vt * kLmTileM, 0, pol_a);
          tma_load_3d(smem + L::kBOff + s * L::kBBytes, &tmB, &full[s], kb * kLmTileK,
                      cb * kLmBlock + h * kLmHalf, 0, pol_b);
        }
      }
      // let every copy this thread issued land before the CTA can exit
      const int first = g > kLmStages ? g - kLmStages : 0;
      for (int x = first; x < g; ++x) {
        int dummy_abort = 0;
        mbar_wait_bounded(&full[x % kLmStages], (x / kLmStages) & 1, &dummy_abort, p.status);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int g = 0, it = 0, n1 = 0;  // n1: tiles that used half 1
      bool ok = true;
      for (int u = u0; ok && u < u1; ++u, ++it) {
        const int cb = u / p.n_vt;
        int ncols, nb0, nb1;
        block_shape(p, cb, ncols, nb0, nb1);
        const uint32_t idesc0 = umma_idesc_bf16(kLmTileM, nb0);
        const uint32_t idesc1 = nb1 > 0 ? umma_idesc_bf16(kLmTileM, nb1) : 0u;
        const int nh = nb1 > 0 ? 2 : 1;
        for (int st = 0; st < nkb * nh; ++st, ++g) {
          const int kb = st / nh, h = st - kb * nh;
          const int s = g % kLmStages;
          if (!mbar_wait_bounded(&full[s], (g / kLmStages) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          // a TMEM half is written again only once the epilogue has read it
          if (kb == 0 && !mbar_wait_bounded(&tempty[h], (h == 0 ? (it & 1) : (n1 & 1)) ^ 1u,
                                            abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + L::kAOff + s * L::kABytes);
          const uint32_t b_addr = smem_u32(smem + L::kBOff + s * L::kBBytes);
          const uint32_t idesc = h == 0 ? idesc0 : idesc1;
#pragma unroll
          for (int kk = 0; kk < kLmTileK / 16; ++kk)
            umma_bf16(tmem_base + h * kLmHalf, umma_desc_sw128(a_addr + kk * 32),
                      umma_desc_sw128(b_addr + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        if (nb1 > 0) ++n1;
        umma_commit(tfull);
      }
      // every MMA this thread issued must finish before TMEM is released
      umma_commit(drain);
      int dummy_abort = 0;
      mbar_wait_bounded(drain, 0, &dummy_abort, p.status);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int te = threadIdx.x - 64;  // 0..127
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    RowPart* red = reinterpret_cast<RowPart*>(smem + L::kRedOff);  // [4][256] per-warp results
    // this warp's 32 x 32 transpose scratch, rows padded to 33 words
    float* tsc = reinterpret_cast<float*>(smem + L::kScrOff) + quad * 32 * 33;
    const bool typical = p.typical != 0;
    // the four epilogue warps synchronise on an mbarrier with a bounded wait
    uint32_t epi_phase = 0;
    bool epi_ok = true;
    auto epi_sync = [&]() {
      mbar_arrive(epi);
      epi_ok = mbar_wait_bounded(epi, epi_phase, abort_flag, p.status);
      epi_phase ^= 1u;
      return epi_ok;
    };
    // the CTA's running records of block-local columns h * 256 + te + 128 k
    RowPart run[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int k = 0; k < 2; ++k) run[h][k] = empty_record();
    bool bad = false;  // a NaN logit
    int it = 0;
    for (int u = u0; epi_ok && u < u1; ++u, ++it) {
      const int cb = u / p.n_vt, vt = u - cb * p.n_vt;
      int ncols, nb0, nb1;
      block_shape(p, cb, ncols, nb0, nb1);
      if (!mbar_wait_bounded(tfull, it & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const int row0 = vt * kLmTileM + quad * 32;  // vocabulary row of this warp's lane 0
      const bool row_ok = row0 + lane < p.V;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int nbh = h ? nb1 : nb0;
        if (!epi_ok || nbh == 0) break;
        const int ngroups = (nbh + 31) / 32;
#pragma unroll 1
        for (int gq = 0; gq < ngroups; ++gq) {
          const int col0 = h * kLmHalf + gq * 32;  // block-local column of z[0]
          float z[32];
          tmem_ld32(tmem_base + lane_off + col0, z);
          if (p.logits != nullptr && row_ok) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < ncols)
                p.logits[(size_t)(cb * kLmBlock + col0 + j) * p.V + row0 + lane] = z[j];
          }
          // transpose through shared memory: lane = row on the way in, lane =
          // column on the way out (padding keeps both directions free of bank
          // conflicts)
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            bad |= row_ok && (col0 + j < ncols) && (z[j] != z[j]);
            tsc[lane * 33 + j] = row_ok ? z[j] : -INFINITY;
          }
          __syncwarp();
          float c[32];
#pragma unroll
          for (int r = 0; r < 32; ++r) c[r] = tsc[r * 33 + lane];
          __syncwarp();
          // column `lane`: largest value, lowest row among equals (four
          // chains over rows r = q, q + 4, ..., then merged in row order)
          float bv[4];
          int br[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            bv[q] = c[q];
            br[q] = q;
          }
#pragma unroll
          for (int r = 4; r < 32; ++r) {
            if (c[r] > bv[r & 3]) {
              bv[r & 3] = c[r];
              br[r & 3] = r;
            }
          }
          float m = bv[0];
          int mr = br[0];
#pragma unroll
          for (int q = 1; q < 4; ++q) {
            if (bv[q] > m || (bv[q] == m && br[q] < mr)) {
              m = bv[q];
              mr = br[q];
            }
          }
          RowPart rec;
          rec.maxz = m;
          rec.idx = m == -INFINITY ? 0x7fffffff : row0 + mr;
          rec.s = 0.f;
          rec.t = 0.f;
          if (typical && m != -INFINITY) {
            float s = 0.f, t = 0.f;
#pragma unroll
            for (int r = 0; r < 32; ++r) {
              const float w = lm_ex2((c[r] - m) * p.t_log2);  // -inf rows give 0
              s += w;
              t += c[r] == -INFINITY ? 0.f : w * (c[r] * p.inv_T);
            }
            rec.s = s;
            rec.t = t;
          }
          red[quad * kLmHalf + gq * 32 + lane] = rec;
        }
        // this half is read: the next tile may overwrite it
        tc_fence_before();
        mbar_arrive(&tempty[h]);
        if (!epi_sync()) break;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int cc = te + 128 * k;
          if (cc < ngroups * 32) {
            RowPart r = red[cc];
#pragma unroll
            for (int q = 1; q < 4; ++q) merge_record(r, red[q * kLmHalf + cc], typical, p.t_log2);
            merge_record(run[h][k], r, typical, p.t_log2);
          }
        }
        if (!epi_sync()) break;
      }
      // last tile of this column block in the CTA's range: write the records
      if (epi_ok && (u + 1 == u1 || (u + 1) / p.n_vt != cb)) {
        const int c_first = (cb * p.n_vt) / p.per;
        const int c_last = (cb * p.n_vt + p.n_vt - 1) / p.per;
        const int slot = static_cast<int>(blockIdx.x) - c_first;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int cc = h * kLmHalf + te + 128 * k;
            if (cc < ncols) {
              RowPart* dst = p.part + (size_t)(cb * kLmBlock + cc) * p.n_slots;
              dst[slot] = run[h][k];
              // the block's last CTA pads its columns' unused record slots
              if (static_cast<int>(blockIdx.x) == c_last)
                for (int s2 = slot + 1; s2 < p.n_slots; ++s2) dst[s2] = empty_record();
            }
            run[h][k] = empty_record();
          }
      }
    }
    if (bad) report(p.status, MEDUSA_ERR_DEVICE_CHECK);
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
    tmem_dealloc(tmem_base, 2 * kLmHalf);
  }
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
namespace {

struct LmPlan {
  int n_vt, n_cb, n_units, per, grid, n_slots;
};

LmPlan lm_plan(int C, int V) {
  LmPlan q{};
  q.n_vt = (V + kLmTileM - 1) / kLmTileM;
  q.n_cb = (C + kLmBlock - 1) / kLmBlock;
  q.n_units = q.n_vt * q.n_cb;
  const int sms = device_sm_count();
  const int g0 = q.n_units < sms ? q.n_units : sms;
  q.per = (q.n_units + g0 - 1) / g0;
  q.grid = (q.n_units + q.per - 1) / q.per;  // every CTA has at least one unit
  q.n_slots = 1;
  for (int cb = 0; cb < q.n_cb; ++cb) {
    const int first = (cb * q.n_vt) / q.per, last = (cb * q.n_vt + q.n_vt - 1) / q.per;
    if (last - first + 1 > q.n_slots) q.n_slots = last - first + 1;
  }
  return q;
}

}  // namespace

size_t lmhead_verify_workspace_size(int B, int N, int d, int V) {
  (void)d;
  const int C = B * N;
  const LmPlan q = lm_plan(C, V);
  return align256((size_t)C * q.n_slots * sizeof(RowPart));
}

medusa_status_t lmhead_verify(const void* hidden, const void* lm_head, const int32_t* cand_ids,
                              const medusa_tree_t& tree, int B, int d, int V,
                              medusa_accept_t mode, float temperature, float eps, float delta,
                              int32_t* accept_len, int32_t* accepted_nodes,
                              int32_t* accepted_tokens, int32_t* bonus, float* logits, void* ws,
                              int32_t* status, cudaStream_t stream) {
  const int N = tree.n_nodes;
  const int C = B * N;
  const LmPlan q = lm_plan(C, V);
  // lm_head [V][d] and hidden [C][d] as 3-D tensors of one plane
  CUtensorMap mA, mB;
  const uint64_t da[3] = {(uint64_t)d, (uint64_t)V, 1};
  const uint64_t sa[2] = {(uint64_t)d * 2, (uint64_t)V * d * 2};
  const uint32_t ba[3] = {kLmTileK, kLmTileM, 1};
  const uint64_t db[3] = {(uint64_t)d, (uint64_t)C, 1};
  const uint64_t sb[2] = {(uint64_t)d * 2, (uint64_t)C * d * 2};
  const uint32_t bb[3] = {kLmTileK, kLmHalf, 1};
  if (!make_tmap_bf16(&mA, lm_head, 3, da, sa, ba) || !make_tmap_bf16(&mB, hidden, 3, db, sb, bb))
    return fail(MEDUSA_ERR_CUDA, "lmhead_verify: cuTensorMapEncodeTiled failed");
  if (cudaFuncSetAttribute(lmhead_reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           LmSmem::kAlloc) != cudaSuccess)
    return fail(MEDUSA_ERR_CUDA, "cudaFuncSetAttribute(lmhead_reduce) failed");
  const bool typical = mode == MEDUSA_ACCEPT_TYPICAL;
  LmParams p{};
  p.V = V;
  p.d = d;
  p.C = C;
  p.n_vt = q.n_vt;
  p.n_cb = q.n_cb;
  p.n_units = q.n_units;
  p.per = q.per;
  p.n_slots = q.n_slots;
  p.typical = typical ? 1 : 0;
  p.inv_T = typical ? 1.0f / temperature : 1.0f;
  p.t_log2 = p.inv_T * 1.4426950408889634f;
  p.logits = logits;
  p.part = static_cast<RowPart*>(ws);
  p.status = status;
  launch(lmhead_reduce_kernel, q.grid, kLmThreads, LmSmem::kAlloc, stream, mA, mB, p);
  medusa_status_t st = check_launch("lmhead_reduce");
  if (st != MEDUSA_OK) return st;
  return verify_path_from_parts(p.part, q.n_slots, static_cast<const __nv_bfloat16*>(hidden),
                                static_cast<const __nv_bfloat16*>(lm_head), d, cand_ids, tree, B,
                                V, mode, temperature, eps, delta, accept_len, accepted_nodes,
                                accepted_tokens, bonus, status, stream);
}

}  // namespace medusa
