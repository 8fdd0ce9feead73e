// k_attn.cu -- block-sparse attention forward over kept 64 x 64 tiles
// (NABLA, Methodology item 2, "expansion": the block mask decides which
// N x N tiles are computed; Sparse VideoGen2 section 2C: contiguous query
// blocks are computed densely while key/value blocks are loaded sparsely).
//
// Blackwell mapping.  A work item is a 128-row query tile made of two 64-token
// query blocks of one (batch, head): the same patch in frames 2t and 2t+1,
// whose kept lists overlap most (time pairing).  The item walks the merged,
// ascending union of both lists two key blocks (128 keys) per step n:
//   S_n = Q K_n^T  tcgen05.mma M=128, N=64*nb, K=d  (SMEM x SMEM -> TMEM S[n%3])
// (N = 128 whenever the step has two blocks: N = 64 MMAs run at ~2/3 rate)
//   P_n = online softmax of S_n, per row only over the blocks its own query
//         block keeps, written as packed bf16 over the first 64 columns of
//         the same TMEM buffer
//   O  += P_n V_n  tcgen05.mma M=128, N=d, K=64*nb  (TMEM x SMEM -> TMEM O)
// Three S buffers let the MMA warp keep the scores up to two steps ahead of
// the softmax: the tensor core runs S_{n+2} while P_n is being formed; S_{n+3}
// reuses step n's buffer only after PV_n has completed.
// Warp roles (384 threads, one CTA per SM, persistent):
//   warp 0      producer: takes items from an atomic counter over a
//               longest-first work list, merges the two CSR lists, publishes
//               one step record per step (8-deep ring) and issues the TMA
//               loads of Q per item and of K per step into a 3-deep ring.
//               Every 64-row block is one 4-D box (64 elements x 8 rows x
//               d/64 halves x 8 row groups), stored 128B-swizzled as
//               [row group][d-half][8 rows][128 B]: the rows of two blocks
//               then sit at one uniform group stride of 16*d bytes (the SBO)
//               and the d-halves 1 KiB apart.  In the raster layout the
//               block is the 8 x 8 patch of its frame, fetched by one 5-D box
//               that lands in the same SMEM order;
//   warp 11     V producer: follows the step records and loads V per step
//               into its own 3-deep ring;
//   warp 1      allocates 512 TMEM columns; one lane issues the S MMAs;
//   warp 10     one lane issues the PV MMAs.  tcgen05.mma issue is paced by
//               the tensor core, so two issuers let one's waits overlap the
//               other's MMAs (commits track each thread's own MMAs);
//   warps 2..9  two softmax warpgroups taking alternate steps (even steps:
//               warps 2..5, odd steps: warps 6..9), one thread per query row:
//               softmax, lazy O rescale (only when the running max grows by
//               more than 2^8), epilogue O / l -> bf16 and LSE.  Only the
//               running max and row sum pass between the two groups.
// TMEM columns: S0 [0,128), S1 [128,256), S2 [256,384), O [384,384+d).
// Every mbarrier wait is bounded; a wait that gives up records an error code
// and the CTA winds down instead of hanging.
#include "vsa_device.cuh"
#include "vsa_internal.h"
#include "vsa_tma.h"

#include <cmath>
#include <cstdio>
#include <mutex>

namespace vsa {
namespace {

constexpr int kThreads = 384;
constexpr int kRing = 3;               // K stages, V stages, S buffers
constexpr int kMetaRing = 8;
constexpr int kListWin = 32;           // CSR entries staged per list in SMEM
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 384;

struct StepMeta {
  int32_t blk0, blk1;  // key blocks of this step (blk1 = -1 when nb == 1)
  int32_t nb;          // 1 or 2 key blocks; 0 = empty item; -1 = no more work
  uint32_t flags;      // bit0/1: blk0 kept by query block 0/1; bit2/3: blk1;
                       // bits 8-14 / 16-22: valid keys of blk0 / blk1 (1..64)
  int32_t bh, r0, r1;  // head slice and query blocks (r1 = -1 if absent)
  int32_t first_last;  // bit0: first step of the item, bit1: last step
  int32_t seq;         // item sequence number within this CTA
};

template <int D>
struct Smem {
  static constexpr int kQBytes = 128 * D * 2;             // two query blocks
  static constexpr int kBlockBytes = 64 * D * 2;          // one 64-row block
  static constexpr int kGroupBytes = 8 * D * 2;            // 8 rows, all d-halves
  static constexpr int kKVBytes = 2 * kBlockBytes;         // K (or V) of two key blocks
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQBytes;
  static constexpr int kVOff = kKOff + kRing * kKVBytes;
  static constexpr int kMetaOff = kVOff + kRing * kKVBytes;
  static constexpr int kListOff = kMetaOff + kMetaRing * static_cast<int>(sizeof(StepMeta));
  static constexpr int kXchgOff = kListOff + 2 * kListWin * 4;   // m_sh[2][128], l_sh[2][128]
  static constexpr int kBarOff = (kXchgOff + 4 * 128 * 4 + 7) & ~7;
  // k_full[3] v_full[3] s_full[3] pv_buf[3] meta_full[8] meta_empty[8]
  // q_full q_empty p_full[4] o_full[0] o_empty m_full[2] l_full[2] o_full[1]
  // (s_full also frees K stages and pv_buf V stages: same completions)
  static constexpr int kNumBars = 4 * kRing + 2 * kMetaRing + 2 + 4 + 3 + 4;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kTmemSlotOff + 16;
  static constexpr int kAlloc = kBytes;                   // base is 1 KiB aligned
  static_assert(kAlloc <= 232448, "shared memory layout exceeds 227 KiB");
};

struct AttnArgs {
  const int64_t *row_ptr;
  const int32_t *col_idx;
  __nv_bfloat16 *o;
  float *lse;
  const int32_t *order;   // longest-first work items
  int *counter;           // next position in `order`
  unsigned *err;
  int64_t items;          // total work items (when n_items is null)
  const int *n_items;     // query-subset mode: item count written by the planner;
                          // order[] then holds the list index of each item's lead
  const int32_t *qblocks; // query-subset mode: the listed global query-block rows
  int64_t n_qblocks;
  const int32_t *kvalid;  // optional: valid keys (1..64) of each key block, the rest
                          // of the block is masked out; null: all 64
  int64_t N;              // tokens per head
  int Nb, T, HW;          // blocks per head, frames, patches per frame
  int H, W, Wb;           // raster rows and columns per frame, patches per row
  uint64_t hw_mul, wb_mul;  // ceil(2^32 / HW), ceil(2^32 / Wb): exact quotients
                            // n / HW and n / Wb as (n * mul) >> 32 while n * HW < 2^32
  int pairs_per_head;
  float c;                // scale * log2(e)
  float lse_scale;        // ln(2)
};

// item -> (bh, r0, r1): the same patch in frames 2t and 2t+1.  In the
// query-subset mode an item is the list index i of its lead block; the next
// listed block joins it when it belongs to the same head and comes after it
// (the planner emits only leads, in range).
__device__ __forceinline__ void decode_item(int item, const AttnArgs &a, int &bh, int &r0,
                                            int &r1) {
  if (a.n_items) {
    const int32_t g0 = a.qblocks[item];
    bh = g0 / a.Nb;
    r0 = g0 % a.Nb;
    const int32_t g1 = item + 1 < a.n_qblocks ? a.qblocks[item + 1] : -1;
    r1 = (g1 > g0 && g1 / a.Nb == bh) ? g1 % a.Nb : -1;
    return;
  }
  bh = item / a.pairs_per_head;
  const int p = item % a.pairs_per_head;
  const int t2 = p / a.HW, sp = p % a.HW;
  r0 = 2 * t2 * a.HW + sp;
  r1 = (2 * t2 + 1 < a.T) ? r0 + a.HW : -1;
}

// Frame and patch of 64-token block r (fractal order: frame-major, then the
// patches of the frame row-major).
__device__ __forceinline__ void block_patch(int r, const AttnArgs &a, int &t, int &py, int &px) {
  t = static_cast<int>((static_cast<uint64_t>(r) * a.hw_mul) >> 32);
  const int sp = r - t * a.HW;
  py = static_cast<int>((static_cast<uint64_t>(sp) * a.wb_mul) >> 32);
  px = sp - py * a.Wb;
}

// TMA load of 64-token block r of head slice bh into one operand stage.
// Flattened layout: the block's 8 row groups are consecutive.  Raster layout:
// the block is the 8 x 8 patch of its frame, so the box is placed by
// (column, row, frame) coordinates and lands in the same SMEM order.
template <bool kRaster>
__device__ __forceinline__ void load_block(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                           const AttnArgs &a, int bh, int r) {
  if constexpr (kRaster) {
    int t, py, px;
    block_patch(r, a, t, py, px);
    tma_load_5d(dst, m, bar, 0, px * 8, 0, py * 8, bh * a.T + t);
  } else {
    tma_load_4d(dst, m, bar, 0, 0, 0, static_cast<int>(static_cast<int64_t>(bh) * a.N / 8) + r * 8);
  }
}

// L2 prefetch of block r of head slice bh (the same box load_block fetches).
template <bool kRaster>
__device__ __forceinline__ void prefetch_block(const CUtensorMap *m, const AttnArgs &a, int bh,
                                               int r) {
  if constexpr (kRaster) {
    int t, py, px;
    block_patch(r, a, t, py, px);
    tma_prefetch_5d(m, 0, px * 8, 0, py * 8, bh * a.T + t);
  } else {
    tma_prefetch_4d(m, 0, 0, 0, static_cast<int>(static_cast<int64_t>(bh) * a.N / 8) + r * 8);
  }
}

// Token index within its head of position i (= 8 * patch row + column) of
// block r.
template <bool kRaster>
__device__ __forceinline__ int64_t block_token(const AttnArgs &a, int r, int i) {
  if constexpr (!kRaster) {
    return static_cast<int64_t>(r) * 64 + i;
  } else {
    int t, py, px;
    block_patch(r, a, t, py, px);
    return (static_cast<int64_t>(t) * a.H + py * 8 + (i >> 3)) * a.W + px * 8 + (i & 7);
  }
}

// One 32-column chunk Q of the softmax's second pass: starts the load of
// chunk Q+1 into `nxt`, exponentiates `cur` (already loaded) against the
// reference, adds to the row sums and stores P as 16 packed bf16x2 columns
// over S columns [16Q, 16Q+16) (scores already read), then waits for `nxt`.
// Chunks 0-1 are key block 0 (valid when v0), chunks 2-3 key block 1.
// `lim` is the number of valid key columns in this chunk (32 unless the key
// block is a partial one); columns past it get P = 0.
template <int Q, bool kKeyMask>
__device__ __forceinline__ void softmax_chunk(uint32_t (&cur)[32], uint32_t (&nxt)[32], int nq,
                                              bool v0, bool v1, uint32_t s_addr, float2 c2,
                                              float2 nm2, float2 (&r4)[4], int lim) {
  if (Q >= nq) return;
  const bool vq = Q < 2 ? v0 : v1;
  const bool vn = Q + 1 < nq && (Q + 1 < 2 ? v0 : v1);
  if (vn) tmem_ld32_nowait(s_addr + 32 * (Q + 1), nxt);
  uint32_t pk[16];
  if (vq && (!kKeyMask || lim >= 32)) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float2 t =
          ffma2(make_float2(__uint_as_float(cur[2 * j]), __uint_as_float(cur[2 * j + 1])), c2, nm2);
      const float2 p = make_float2(ex2(t.x), ex2(t.y));
      r4[j & 3] = fadd2(r4[j & 3], p);
      pk[j] = pack_bf16x2(p.x, p.y);
    }
  } else if (kKeyMask && vq) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float2 t =
          ffma2(make_float2(__uint_as_float(cur[2 * j]), __uint_as_float(cur[2 * j + 1])), c2, nm2);
      const float2 p = make_float2(2 * j < lim ? ex2(t.x) : 0.0f,
                                   2 * j + 1 < lim ? ex2(t.y) : 0.0f);
      r4[j & 3] = fadd2(r4[j & 3], p);
      pk[j] = pack_bf16x2(p.x, p.y);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) pk[j] = 0u;
  }
  tmem_st16u(s_addr + 16 * Q, pk);
  if (vn) tmem_wait_ld_regs(nxt);
}

// kKeyMask: key blocks may be partial (per-block valid counts in AttnArgs);
// the plain instantiation carries no masking code.  kLayout 0: Q, K, V, O and
// LSE in the flattened (fractal) token order; 1: all in raster order (blocks
// fetched as patches); 2: Q, K, V flattened, O and LSE stored in raster order
// (the unflatten of the output folded into the epilogue's row addresses).
template <int D, bool kKeyMask, int kLayout>
__global__ void __maxnreg__(168)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tq,
                       const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const AttnArgs a) {
  using L = Smem<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // The 128B-swizzled operand tiles need a 1 KiB aligned base; if the
  // dynamic allocation is not aligned, every thread leaves before touching
  // barriers, TMEM or TMA (uniform exit, recorded in the error word).
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(a.err, kErrSmemAlign);
    return;
  }
  unsigned char *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  StepMeta *meta = reinterpret_cast<StepMeta *>(smem + L::kMetaOff);
  int32_t *list0 = reinterpret_cast<int32_t *>(smem + L::kListOff);
  int32_t *list1 = list0 + kListWin;
  float *m_sh = reinterpret_cast<float *>(smem + L::kXchgOff);   // [2][128]
  float *l_sh = m_sh + 256;                                        // [2][128]
  const uint32_t bar = sbase + L::kBarOff;
  auto k_full = [&](int s) { return bar + 8u * s; };
  auto v_full = [&](int s) { return bar + 8u * (kRing + s); };
  auto s_full = [&](int s) { return bar + 8u * (2 * kRing + s); };
  auto pv_buf = [&](int s) { return bar + 8u * (3 * kRing + s); };
  auto meta_full = [&](int s) { return bar + 8u * (4 * kRing + s); };
  auto meta_empty = [&](int s) { return bar + 8u * (4 * kRing + kMetaRing + s); };
  const uint32_t q_full = bar + 8u * (4 * kRing + 2 * kMetaRing);
  const uint32_t q_empty = q_full + 8;
  auto p_full = [&](int s) { return q_full + 16u + 8u * s; };   // 4 slots
  // O complete, one barrier per item parity: item s completes phase s/2 of
  // o_full(s & 1), so the phase before the one an epilogue waits for belongs
  // to item s - 2, which is ordered before it (see the epilogue's wait)
  auto o_full = [&](int s) { return s ? q_full + 96u : q_full + 48u; };
  const uint32_t o_empty = q_full + 56;
  auto m_full = [&](int s) { return q_full + 64u + 8u * s; };
  auto l_full = [&](int s) { return q_full + 80u + 8u * s; };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kTmemSlotOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(s_full(s), 1);
      mbar_init(pv_buf(s), 1);
    }
    for (int s = 0; s < kMetaRing; ++s) {
      mbar_init(meta_full(s), 1);
      mbar_init(meta_empty(s), 4);        // one arrival per softmax warp
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 4; ++s) mbar_init(p_full(s), 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(m_full(s), 4);            // one arrival per softmax warp
      mbar_init(l_full(s), 4);
    }
    mbar_init(o_full(0), 1);
    mbar_init(o_full(1), 1);
    mbar_init(o_empty, 128);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
    }
    const int64_t n_items = a.n_items ? static_cast<int64_t>(*a.n_items) : a.items;
    int m = 0;               // next step whose record and K blocks go out
    uint32_t q_phase = 0;
    bool ok = true;
    int nitems = 0;
    // Publishes step record r as step m and loads its K blocks (one 4-D box
    // per block, row-group-major in the stage).
    auto emit = [&](const StepMeta &r) -> bool {
      const int s3 = m % kRing, sm = m % kMetaRing;
      if (!mbar_wait(meta_empty(sm), ((m / kMetaRing) & 1) ^ 1, a.err, kErrWaitSoftmax)) return false;
      // the stage's previous user S_{m-3} has completed (its s_full)
      if (m >= kRing && !mbar_wait(s_full(s3), ((m - kRing) / kRing) & 1, a.err, kErrWaitMma))
        return false;
      if (lane == 0) {
        meta[sm] = r;
        mbar_arrive(meta_full(sm));
        const int nb = r.nb > 0 ? r.nb : 0;
        const uint32_t kf = k_full(s3);
        mbar_arrive_expect_tx(kf, static_cast<uint32_t>(nb * L::kBlockBytes));
        const uint32_t kbase = sbase + L::kKOff + s3 * L::kKVBytes;
        if (nb > 0) load_block<kLayout == 1>(kbase, &tk, kf, a, r.bh, r.blk0);
        if (nb > 1) load_block<kLayout == 1>(kbase + L::kBlockBytes, &tk, kf, a, r.bh, r.blk1);
      }
      __syncwarp();
      ++m;
      return true;
    };
    // The next item's header is fetched one dependent load per emitted step
    // (work counter -> plan entry -> row pointers -> first list windows, and
    // an L2 prefetch of its Q blocks), so item starts do not stall the
    // producer on a chain of global round trips.  hs: 0 nothing fetched,
    // 1 counter value pending, 2 plan entry pending, 3 row pointers pending,
    // 4 ready, 5 no more work.
    int hs = 0;
    int h_raw = 0, h_item = 0, h_bh = 0, h_r0 = 0, h_r1 = -1;
    int64_t h_rp0 = 0, h_rp1 = 0, h_rp2 = 0, h_rp3 = 0;
    int h_pre0 = 0, h_pre1 = 0;      // this lane's entry of each list's first window
    auto advance = [&]() {
      if (hs == 0) {
        if (lane == 0) h_raw = atomicAdd(a.counter, 1);
        hs = 1;
      } else if (hs == 1) {
        h_raw = __shfl_sync(0xFFFFFFFFu, h_raw, 0);
        if (h_raw >= n_items) {
          hs = 5;
        } else {
          h_item = a.order[h_raw];
          hs = 2;
        }
      } else if (hs == 2) {
        decode_item(h_item, a, h_bh, h_r0, h_r1);
        const int64_t g0 = static_cast<int64_t>(h_bh) * a.Nb + h_r0;
        h_rp0 = a.row_ptr[g0];
        h_rp1 = a.row_ptr[g0 + 1];
        if (h_r1 >= 0) {
          const int64_t g1 = static_cast<int64_t>(h_bh) * a.Nb + h_r1;
          h_rp2 = a.row_ptr[g1];
          h_rp3 = a.row_ptr[g1 + 1];
        }
        hs = 3;
      } else if (hs == 3) {
        const int64_t n0 = h_rp1 - h_rp0, n1 = h_r1 >= 0 ? h_rp3 - h_rp2 : 0;
        h_pre0 = lane < n0 ? a.col_idx[h_rp0 + lane] : 0;
        h_pre1 = lane < n1 ? a.col_idx[h_rp2 + lane] : 0;
        if (lane == 0) {
          prefetch_block<kLayout == 1>(&tq, a, h_bh, h_r0);
          if (h_r1 >= 0) prefetch_block<kLayout == 1>(&tq, a, h_bh, h_r1);
        }
        hs = 4;
      }
    };
    while (hs < 4) advance();
    while (ok) {
      if (hs == 5) {
        // one end record per softmax group (they take alternate steps), then
        // the V blocks still owed
        StepMeta r{};
        r.nb = -1;
        if (emit(r)) emit(r);
        break;
      }
      const int bh = h_bh, r0 = h_r0, r1 = h_r1;
      const int64_t b0 = h_rp0, n0 = h_rp1 - h_rp0;
      const int64_t b1 = r1 >= 0 ? h_rp2 : 0, n1 = r1 >= 0 ? h_rp3 - h_rp2 : 0;
      // first windows from the prefetched entries; the next windows' entries
      // are loaded into registers one window ahead
      __syncwarp();
      if (lane < kListWin) {
        list0[lane] = h_pre0;
        list1[lane] = h_pre1;
      }
      __syncwarp();
      int nx0 = lane < n0 - kListWin ? a.col_idx[b0 + kListWin + lane] : 0;
      int nx1 = lane < n1 - kListWin ? a.col_idx[b1 + kListWin + lane] : 0;
      hs = 0;                          // start on the following item's header
      // Q tile: query block r0 -> rows 0..63, r1 -> rows 64..127
      if (nitems > 0) {
        if (!mbar_wait(q_empty, q_phase, a.err, kErrWaitMma)) break;
        q_phase ^= 1u;
      }
      ++nitems;
      if (lane == 0) {
        const int nq = r1 >= 0 ? 2 : 1;
        mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(nq * 64 * D * 2));
        for (int j = 0; j < nq; ++j)
          load_block<kLayout == 1>(sbase + L::kQOff + j * L::kBlockBytes, &tq, q_full, a, bh, j ? r1 : r0);
      }
      // merge the two ascending lists, two union entries per step
      const int64_t g0 = static_cast<int64_t>(bh) * a.Nb + r0;
      int64_t i0 = 0, i1 = 0, w0 = 0, w1 = 0;
      StepMeta pend{};
      pend.bh = bh; pend.r0 = r0; pend.r1 = r1;
      pend.seq = nitems - 1;
      pend.nb = 0; pend.first_last = 1;
      bool have_pending = false;
      StepMeta cur = pend;
      cur.nb = 0; cur.flags = 0; cur.blk0 = cur.blk1 = -1;
      while (i0 < n0 || i1 < n1) {
        if (i0 < n0 && i0 >= w0 + kListWin) {
          w0 += kListWin;
          __syncwarp();
          if (lane < kListWin) list0[lane] = nx0;
          __syncwarp();
          nx0 = lane < n0 - w0 - kListWin ? a.col_idx[b0 + w0 + kListWin + lane] : 0;
        }
        if (i1 < n1 && i1 >= w1 + kListWin) {
          w1 += kListWin;
          __syncwarp();
          if (lane < kListWin) list1[lane] = nx1;
          __syncwarp();
          nx1 = lane < n1 - w1 - kListWin ? a.col_idx[b1 + w1 + kListWin + lane] : 0;
        }
        const int c0 = i0 < n0 ? list0[i0 - w0] : 0x7FFFFFFF;
        const int c1 = i1 < n1 ? list1[i1 - w1] : 0x7FFFFFFF;
        const int c = c0 < c1 ? c0 : c1;
        const uint32_t f = (c0 == c ? 1u : 0u) | (c1 == c ? 2u : 0u);
        i0 += (c0 == c);
        i1 += (c1 == c);
        if (c < 0 || c >= a.Nb) {  // invalid index: skip it, record once
          if (lane == 0) atomicOr(a.err, kErrBadIndex);
          continue;
        }
        const uint32_t kv = kKeyMask ? static_cast<uint32_t>(a.kvalid[g0 - r0 + c]) & 0x7Fu : 64u;
        if (cur.nb == 0) {
          cur.blk0 = c;
          cur.flags = f | (kv << 8);
          cur.nb = 1;
        } else {
          cur.blk1 = c;
          cur.flags |= (f << 2) | (kv << 16);
          cur.nb = 2;
          if (have_pending) {
            if (!(ok = emit(pend))) break;
            advance();
          }
          pend = cur;
          pend.first_last = have_pending ? 0 : 1;
          have_pending = true;
          cur.nb = 0; cur.flags = 0; cur.blk0 = cur.blk1 = -1;
        }
      }
      if (!ok) break;
      if (cur.nb > 0) {
        if (have_pending) {
          if (!(ok = emit(pend))) break;
          advance();
        }
        const int first = have_pending ? 0 : 1;
        pend = cur;
        pend.first_last = first;
        have_pending = true;
      }
      if (!have_pending) {  // empty item: one step without blocks
        pend.nb = 0; pend.flags = 0; pend.blk0 = pend.blk1 = -1;
        pend.first_last = 1;
      }
      pend.first_last |= 2;
      if (!(ok = emit(pend))) break;
      while (hs < 4) advance();        // short items: finish the next header now
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer
    uint32_t q_phase = 0;
    constexpr uint32_t kIdescS1 = idesc_bf16(128, 64, false, false);
    constexpr uint32_t kIdescS2 = idesc_bf16(128, 128, false, false);
    constexpr uint32_t kStageUnits = L::kKVBytes >> 4;   // one stage in 16-byte units
    // Descriptors are built once; per MMA only the 14-bit start-address field
    // (16-byte units, low word) moves.
    const uint64_t q_desc = smem_desc(sbase + L::kQOff, 16, L::kGroupBytes);
    const uint64_t k_desc0 = smem_desc(sbase + L::kKOff, 16, L::kGroupBytes);
    for (int n = 0;; ++n) {
      const int b = n % kRing;
      if (!mbar_wait(k_full(b), (n / kRing) & 1, a.err, kErrWaitTma)) break;
      const StepMeta r = meta[n % kMetaRing];
      if (r.nb < 0) break;
      // S_n overwrites the buffer whose first columns held P_{n-3}: PV_{n-3}
      // must have finished reading it (consecutive MMAs overlap in the pipe).
      // At most PV_{n-3} can have completed into this buffer yet, so the
      // parity names it exactly.
      if (n >= kRing && !mbar_wait(pv_buf(b), ((n - kRing) / kRing) & 1, a.err, kErrWaitMma)) break;
      if (r.first_last & 1) {
        if (!mbar_wait(q_full, q_phase, a.err, kErrWaitTma)) break;
        q_phase ^= 1u;
      }
      tc_fence_after();
      if (lane == 0) {
        if (r.nb > 0) {
          // one chain, N = 64*nb: both blocks' rows at the uniform group stride
          const uint64_t kd = k_desc0 + static_cast<uint32_t>(b) * kStageUnits;
          const uint32_t dcol = tmem + static_cast<uint32_t>(b) * 128u;
          const uint32_t idesc_s = r.nb > 1 ? kIdescS2 : kIdescS1;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            // k-th 16-column slice: 32 B inside the 128 B swizzle row, d-halves 1 KiB apart
            const uint32_t off = (k >> 2) * 64 + (k & 3) * 2;
            mma_bf16_ss(dcol, q_desc + off, kd + off, idesc_s, k > 0);
          }
        }
        mma_commit(s_full(b));          // also frees K stage b
        if (r.first_last & 2) mma_commit(q_empty);
      }
      __syncwarp();
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ PV issuer
    uint32_t oe_phase = 0;
    bool first_item = true;
    constexpr uint32_t kIdescO = idesc_bf16(128, D, false, true);
    constexpr uint32_t kStageUnits = L::kKVBytes >> 4;
    // V is an MN-major operand: 8-key groups kGroupBytes apart (SBO, across
    // both blocks), d-halves 1 KiB apart (LBO)
    const uint64_t v_desc0 = smem_desc(sbase + L::kVOff, 1024, L::kGroupBytes);
    constexpr uint32_t kKStep = (2 * L::kGroupBytes) >> 4;   // 16 keys
    for (int n = 0;; ++n) {
      const int b = n % kRing;
      // the step record tells an end record apart (no P will come); slot n%8
      // is rewritten only for step n+8, after S_{n+5}, which waits for PV_{n+2}
      if (!mbar_wait(meta_full(n % kMetaRing), (n / kMetaRing) & 1, a.err, kErrWaitTma)) break;
      const StepMeta r = meta[n % kMetaRing];
      if (r.nb < 0) break;
      // 4 slots: step n+4 needs S_{n+4}, issued only after PV_{n+1}, so this
      // barrier is never two phases ahead of the wait
      if (!mbar_wait(p_full(n & 3), (n >> 2) & 1, a.err, kErrWaitSoftmax)) break;
      if (r.first_last & 1) {
        if (!first_item) {
          if (!mbar_wait(o_empty, oe_phase, a.err, kErrWaitSoftmax)) break;
          oe_phase ^= 1u;
        }
        first_item = false;
      }
      if (!mbar_wait(v_full(b), (n / kRing) & 1, a.err, kErrWaitTma)) break;
      tc_fence_after();
      if (lane == 0) {
        if (r.nb > 0) {
          const uint64_t vd = v_desc0 + static_cast<uint32_t>(b) * kStageUnits;
          const uint32_t pcol = tmem + static_cast<uint32_t>(b) * 128u;   // P_n in S[n%3]
          const bool acc0 = !(r.first_last & 1);
          // 16 keys per MMA: 8 TMEM columns of P, 2 KiB of V
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16_ts(tmem + kColO, pcol + k * 8, vd + k * kKStep, kIdescO, acc0 || k > 0);
          if (r.nb > 1) {
#pragma unroll
            for (int k = 4; k < 8; ++k)
              mma_bf16_ts(tmem + kColO, pcol + k * 8, vd + k * kKStep, kIdescO, true);
          }
        }
        // O complete before the step's own commit: every later pv_buf
        // arrival then follows this item's O-complete arrival
        if (r.first_last & 2) mma_commit(o_full(r.seq & 1));
        mma_commit(pv_buf(b));          // also frees V stage b
      }
      __syncwarp();
    }
  } else if (warp == 11) {
    // ------------------------------------------------------------ V producer
    if (lane == 0) tma_prefetch_desc(&tv);
    for (int n = 0;; ++n) {
      const int b = n % kRing;
      // slot n%8 is rewritten only for step n+8, after S_{n+5}, which waits
      // for PV_{n+2}, which needs this warp's V_{n+2}
      if (!mbar_wait(meta_full(n % kMetaRing), (n / kMetaRing) & 1, a.err, kErrWaitTma)) break;
      const StepMeta r = meta[n % kMetaRing];
      if (r.nb < 0) break;
      // the stage's previous user PV_{n-3} has completed (its pv_buf)
      if (n >= kRing && !mbar_wait(pv_buf(b), ((n - kRing) / kRing) & 1, a.err, kErrWaitMma)) break;
      if (lane == 0) {
        const int nb = r.nb > 0 ? r.nb : 0;
        const uint32_t vf = v_full(b);
        mbar_arrive_expect_tx(vf, static_cast<uint32_t>(nb * L::kBlockBytes));
        const uint32_t vbase = sbase + L::kVOff + b * L::kKVBytes;
        if (nb > 0) load_block<kLayout == 1>(vbase, &tv, vf, a, r.bh, r.blk0);
        if (nb > 1) load_block<kLayout == 1>(vbase + L::kBlockBytes, &tv, vf, a, r.bh, r.blk1);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int grp = (warp - 2) >> 2;          // 0: even steps, 1: odd steps
    const int quarter = warp & 3;              // TMEM lane quarter of this warp
    const int row = quarter * 32 + lane;       // query row within the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t sel = row >= 64 ? 1u : 0u;
    const float2 c2 = make_float2(a.c, a.c);
    // This group's partial row sum over its own steps of the current item, in
    // the scale of the reference it used last (m_own).  The two partial sums
    // meet only at the item's last step.
    float l_own = 0.0f, m_own = -INFINITY;
    int seq_own = -1;
    for (int n = grp;; n += 2) {
      const int sm = n % kMetaRing;
      if (!mbar_wait(meta_full(sm), (n / kMetaRing) & 1, a.err, kErrWaitTma)) break;
      const StepMeta m = meta[sm];
      __syncwarp();
      if (lane == 0) mbar_arrive(meta_empty(sm));
      if (m.nb < 0) break;
      const bool first = m.first_last & 1, last = m.first_last & 2;
      const int sb = n % kRing;
      const uint32_t s_addr = lane_addr + static_cast<uint32_t>(sb) * 128u;
      if (!mbar_wait(s_full(sb), (n / kRing) & 1, a.err, kErrWaitMma)) break;
      tc_fence_after();
      // warps hold rows of one query block, so v0 / v1 are warp-uniform
      const bool v0 = m.nb > 0 && ((m.flags >> sel) & 1u);
      const bool v1 = m.nb > 1 && ((m.flags >> (2 + sel)) & 1u);
      const int kv0 = static_cast<int>((m.flags >> 8) & 0x7Fu);    // valid keys per block
      const int kv1 = static_cast<int>((m.flags >> 16) & 0x7Fu);
      float mx = -INFINITY;
      if (v0 || v1) {
        // pass 1: row max over the valid halves, 64 scores live at a time
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h ? v1 : v0) {
            float x[64];
            tmem_ld64(s_addr + 64 * h, x);
            const int kv = h ? kv1 : kv0;
            if (kKeyMask && kv < 64) {
#pragma unroll
              for (int j = 0; j < 64; ++j) x[j] = j < kv ? x[j] : -INFINITY;
            }
#pragma unroll
            for (int j = 0; j < 64; j += 2)
              m4[(j >> 1) & 3] = fmax3(m4[(j >> 1) & 3], x[j], x[j + 1]);
          }
        }
        mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * a.c;
      }
      // running max of the previous step (the other group); every step waits
      // for it so that the hand-off barriers stay in lock step
      float m_prev = -INFINITY;
      if (n > 0) {
        if (!mbar_wait(m_full((n - 1) & 1), ((n - 1) >> 1) & 1, a.err, kErrWaitSoftmax)) break;
        if (!first) m_prev = m_sh[((n - 1) & 1) * 128 + row];
      }
      // At the item's last step, take the other group's partial sum (posted
      // at step n-1, in the scale m_prev) before this step's max is posted:
      // the other group writes that slot again only at step n+1, after it has
      // seen this step's max, so the slot cannot be overwritten under us.
      float l_other = 0.0f;
      if (last && !first) {
        if (!mbar_wait(l_full((n - 1) & 1), ((n - 1) >> 1) & 1, a.err, kErrWaitSoftmax)) break;
        l_other = l_sh[((n - 1) & 1) * 128 + row];
      }
      // lazy rescale: move the reference max only when it grows by > 8 (2^8)
      float m_run = m_prev, alpha = 1.0f;
      bool resc = false;
      if (mx > m_prev + 8.0f) {
        if (m_prev != -INFINITY) {
          alpha = ex2(m_prev - mx);
          resc = true;
        }
        m_run = mx;
      }
      m_sh[(n & 1) * 128 + row] = m_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(m_full(n & 1));
      const float mref = m_run == -INFINITY ? 0.0f : m_run;
      const float2 nm2 = make_float2(-mref, -mref);
      // pass 2 over 32-column chunks: chunk q+1 is loaded while chunk q is
      // exponentiated; P of chunk q (16 packed columns) goes to S columns
      // [16q, 16q+16), which hold scores already read
      float2 r4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
      {
        const int nq = 2 * (m.nb > 0 ? m.nb : 0);
        uint32_t xa[32], xb[32];
        if (nq > 0 && v0) {
          tmem_ld32_nowait(s_addr, xa);
          tmem_wait_ld_regs(xa);
        }
        softmax_chunk<0, kKeyMask>(xa, xb, nq, v0, v1, s_addr, c2, nm2, r4, kv0);
        softmax_chunk<1, kKeyMask>(xb, xa, nq, v0, v1, s_addr, c2, nm2, r4, kv0 - 32);
        softmax_chunk<2, kKeyMask>(xa, xb, nq, v0, v1, s_addr, c2, nm2, r4, kv1);
        softmax_chunk<3, kKeyMask>(xb, xa, nq, v0, v1, s_addr, c2, nm2, r4, kv1 - 32);
      }
      const float rs = ((r4[0].x + r4[0].y) + (r4[1].x + r4[1].y)) +
                       ((r4[2].x + r4[2].y) + (r4[3].x + r4[3].y));
      // this group's partial sum, moved to the reference m_run
      if (m.seq != seq_own) {
        l_own = 0.0f;
        seq_own = m.seq;
      } else if (l_own > 0.0f && m_run != m_own) {
        l_own *= ex2(m_own - m_run);
      }
      l_own += rs;
      m_own = m_run;
      l_sh[(n & 1) * 128 + row] = l_own;
      __syncwarp();
      if (lane == 0) mbar_arrive(l_full(n & 1));
      if (__any_sync(0xFFFFFFFFu, resc)) {
        // O must hold PV_{n-1} before it is rescaled.  S_n was issued only
        // after PV_{n-3} completed, so buffer (n-1)%3 has finished every PV
        // before PV_{n-1} and the parity names PV_{n-1} exactly.
        if (!mbar_wait(pv_buf((n - 1) % kRing), ((n - 1) / kRing) & 1, a.err, kErrWaitMma)) break;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < D; cc += 32) {
          float ov[32];
          tmem_ld32(lane_addr + kColO + cc, ov);
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] *= alpha;
          tmem_st32(lane_addr + kColO + cc, ov);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(n & 3));
      if (last) {
        // total row sum in the final reference m_run; the other group's part
        // is in the scale of step n-1's reference m_prev <= m_run
        float l_run = l_own;
        if (l_other > 0.0f) l_run += l_other * ex2(m_prev - m_run);
        // Item seq is phase seq/2 of o_full(seq & 1).  The parity wait can
        // only be early if that barrier's previous phase, item seq - 2, were
        // still open.  It is not: if item seq - 2 ended at step n - 2, this
        // group ran its epilogue and saw that phase complete; if it ended at
        // step n - 3 or before, S_n waited for PV_(n-3)'s commit, which the PV
        // issuer made after item seq - 2's O-complete commit.
        if (!mbar_wait(o_full(m.seq & 1), (static_cast<uint32_t>(m.seq) >> 1) & 1u, a.err,
                       kErrWaitMma))
          break;
        tc_fence_after();
        const int rblk = sel ? m.r1 : m.r0;
        const bool store = rblk >= 0;
        const bool has_keys = l_run > 0.0f;
        const float inv = has_keys ? 1.0f / l_run : 0.0f;
        const int64_t tok =
            static_cast<int64_t>(m.bh) * a.N + (store ? block_token<kLayout != 0>(a, rblk, row & 63) : 0);
        uint4 *orow = reinterpret_cast<uint4 *>(a.o + tok * D);
        // the whole row of O as packed bf16 first; O is then released to the
        // next item's PV MMAs before the global stores go out
        uint32_t pk[D / 2];
#pragma unroll
        for (int cc = 0; cc < D; cc += 32) {
          float ov[32];
          tmem_ld32(lane_addr + kColO + cc, ov);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            pk[cc / 2 + j] = has_keys ? pack_bf16x2(ov[2 * j] * inv, ov[2 * j + 1] * inv) : 0u;
        }
        tc_fence_before();
        mbar_arrive(o_empty);
        if (store) {
#pragma unroll
          for (int j = 0; j < D / 8; ++j)
            orow[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          a.lse[tok] = has_keys ? (m_run + log2f(l_run)) * a.lse_scale : -INFINITY;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Work list: per head, items sorted by descending cost (kept blocks of both
// query blocks), heads in order so that each head's K/V stays L2-resident.
// One CTA per head; also resets the scheduler counter.
__global__ void __launch_bounds__(1024) plan_kernel(const int64_t *__restrict__ row_ptr, int Nb,
                                                    int T, int HW, int pairs, int32_t *order,
                                                    int *counter) {
  extern __shared__ unsigned long long keys[];
  const int bh = blockIdx.x;
  if (bh == 0 && threadIdx.x == 0) *counter = 0;
  int n2 = 1;
  while (n2 < pairs) n2 <<= 1;
  for (int p = threadIdx.x; p < n2; p += blockDim.x) {
    unsigned long long k = ~0ull;
    if (p < pairs) {
      const int t2 = p / HW, sp = p % HW;
      const int r0 = 2 * t2 * HW + sp;
      const int64_t g = static_cast<int64_t>(bh) * Nb + r0;
      int64_t cost = row_ptr[g + 1] - row_ptr[g];
      if (2 * t2 + 1 < T) cost += row_ptr[g + HW + 1] - row_ptr[g + HW];
      if (cost > 0x7FFFFFFF) cost = 0x7FFFFFFF;
      k = (static_cast<unsigned long long>(0x7FFFFFFFu - static_cast<uint32_t>(cost)) << 32) |
          static_cast<uint32_t>(p);
    }
    keys[p] = k;
  }
  __syncthreads();
  for (int size = 2; size <= n2; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const unsigned long long x = keys[i], y = keys[j];
          if ((x > y) == up) {
            keys[i] = y;
            keys[j] = x;
          }
        }
      }
      __syncthreads();
    }
  for (int p = threadIdx.x; p < pairs; p += blockDim.x)
    order[static_cast<int64_t>(bh) * pairs + p] =
        bh * pairs + static_cast<int32_t>(keys[p] & 0xFFFFFFFFu);
}

// Query-subset planner: the listed query blocks (global rows, strictly
// ascending) are paired in list order within each head -- the block of even
// rank within its head leads an item, the next one joins it -- so every item
// but a head's last fills the 128-row tile.  An entry out of range or out of
// order is recorded in the error word and not emitted (the set then computed
// is unspecified, every access stays in bounds).  *n_items starts at zero.
__global__ void plan_rows_kernel(const int32_t *__restrict__ qblocks, int64_t n, int64_t rows,
                                 int Nb, int32_t *order, int *n_items, unsigned *err) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int32_t g = qblocks[i];
  if (g < 0 || g >= rows || (i > 0 && qblocks[i - 1] >= g)) {
    atomicOr(err, kErrBadIndex);
    return;
  }
  // rank of the entry within its head: index minus the head's first entry
  const int32_t head0 = (g / Nb) * Nb;
  int64_t lo = 0, hi = n;
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if (qblocks[mid] < head0) lo = mid + 1; else hi = mid;
  }
  if ((i - lo) & 1) return;        // the second block of its item
  const int pos = atomicAdd(n_items, 1);
  order[pos] = static_cast<int32_t>(i);
}

// Fallback order (no per-head sort) for heads with more than 4096 query-tile
// pairs, beyond the planner's single-CTA bitonic sort.
__global__ void identity_order_kernel(int32_t *order, int64_t n, int *counter) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i == 0) *counter = 0;
  if (i < n) order[i] = static_cast<int32_t>(i);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).

struct AttnLayout {
  int pairs, HW;
  int64_t items;
  size_t order_off, counter_off, total;
};

AttnLayout attn_layout(const Geometry &g) {
  AttnLayout L;
  L.HW = g.Hb * g.Wb;
  L.pairs = ((g.T + 1) / 2) * L.HW;
  L.items = g.BH * L.pairs;
  L.counter_off = 0;      // scheduler counter, then the query-subset item count
  L.order_off = 256;
  L.total = L.order_off + ((static_cast<size_t>(L.items) * 4 + 255) & ~static_cast<size_t>(255));
  return L;
}

}  // namespace

size_t sparse_attn_workspace_bytes(const Geometry &g) { return attn_layout(g).total; }

cudaError_t launch_sparse_attn(const void *qf, const void *kf, const void *vf,
                               const int64_t *row_ptr, const int32_t *col_idx,
                               const Geometry &g, float scale, void *o, float *lse, void *ws,
                               unsigned *err, cudaStream_t st, const char **why,
                               const int32_t *qblocks, int64_t n_qblocks,
                               const int32_t *kvalid, int layout) {
  const bool raster = layout == 1;          // raster loads
  const bool raster_out = layout != 0;      // raster O and LSE
  const AttnLayout L = attn_layout(g);
  if (L.items == 0 || (qblocks && n_qblocks == 0)) return cudaSuccess;
  if (L.items > 0x7FFFFFFF || g.BH * g.N > 0x7FFFFFFF) {
    *why = "sparse attention: too many tokens for 32-bit TMA row coordinates";
    return cudaErrorInvalidValue;
  }
  if (raster_out && g.Nb * L.HW >= (1LL << 32)) {
    *why = "sparse attention: too many blocks per head for the raster layout";
    return cudaErrorInvalidValue;
  }
  const bool masked = kvalid != nullptr;
  if (raster_out && masked) {
    *why = "sparse attention: key masking is not available in the raster layout";
    return cudaErrorInvalidValue;
  }
  CUtensorMap mq, mk, mv;
  const int64_t rows = g.BH * g.N;
  const auto map = [&](CUtensorMap *m, const void *base) {
    return raster ? make_map_raster(m, base, g.BH * g.T, g.H, g.W, g.d)
                  : make_map4(m, base, rows, g.d);
  };
  if (!map(&mq, qf) || !map(&mk, kf) || !map(&mv, vf)) {
    *why = "sparse attention: cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  unsigned char *w = static_cast<unsigned char *>(ws);
  int *counter = reinterpret_cast<int *>(w + L.counter_off);
  int32_t *order = reinterpret_cast<int32_t *>(w + L.order_off);
  int *n_items = counter + 1;
  int n2 = 1;
  while (n2 < L.pairs) n2 <<= 1;
  cudaError_t e;
  if (qblocks) {
    if ((e = cudaMemsetAsync(counter, 0, 2 * sizeof(int), st)) != cudaSuccess) return e;
    plan_rows_kernel<<<static_cast<int>((n_qblocks + 255) / 256), 256, 0, st>>>(
        qblocks, n_qblocks, g.BH * g.Nb, static_cast<int>(g.Nb), order, n_items, err);
  } else if (n2 <= 4096) {
    plan_kernel<<<static_cast<int>(g.BH), 1024, n2 * 8, st>>>(row_ptr, static_cast<int>(g.Nb),
                                                              g.T, L.HW, L.pairs, order, counter);
  } else {
    identity_order_kernel<<<static_cast<int>((L.items + 255) / 256), 256, 0, st>>>(order, L.items,
                                                                                 counter);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  AttnArgs a;
  a.row_ptr = row_ptr; a.col_idx = col_idx;
  a.o = static_cast<__nv_bfloat16 *>(o); a.lse = lse;
  a.order = order; a.counter = counter; a.err = err;
  a.items = L.items; a.N = g.N; a.Nb = static_cast<int>(g.Nb); a.T = g.T; a.HW = L.HW;
  a.H = g.H; a.W = g.W; a.Wb = g.Wb;
  a.hw_mul = ((1ull << 32) + L.HW - 1) / L.HW;
  a.wb_mul = ((1ull << 32) + g.Wb - 1) / g.Wb;
  a.n_items = qblocks ? n_items : nullptr;
  a.qblocks = qblocks;
  a.n_qblocks = n_qblocks;
  a.kvalid = kvalid;
  a.pairs_per_head = L.pairs;
  a.c = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  a.lse_scale = 0.6931471805599453f;
  int grid = num_sms();
  const int64_t max_items = qblocks ? (n_qblocks < L.items ? n_qblocks : L.items) : L.items;
  if (max_items < grid) grid = static_cast<int>(max_items);
  // four instantiations per d: flattened, flattened with key masking (the
  // cluster path), raster, flattened in with raster O and LSE out
  const void *fn;
  int smem;
  if (g.d == 128) {
    fn = masked       ? reinterpret_cast<const void *>(sparse_attn_kernel<128, true, 0>)
         : raster     ? reinterpret_cast<const void *>(sparse_attn_kernel<128, false, 1>)
         : raster_out ? reinterpret_cast<const void *>(sparse_attn_kernel<128, false, 2>)
                      : reinterpret_cast<const void *>(sparse_attn_kernel<128, false, 0>);
    smem = Smem<128>::kAlloc;
  } else {
    fn = masked       ? reinterpret_cast<const void *>(sparse_attn_kernel<64, true, 0>)
         : raster     ? reinterpret_cast<const void *>(sparse_attn_kernel<64, false, 1>)
         : raster_out ? reinterpret_cast<const void *>(sparse_attn_kernel<64, false, 2>)
                      : reinterpret_cast<const void *>(sparse_attn_kernel<64, false, 0>);
    smem = Smem<64>::kAlloc;
  }
  if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
      cudaSuccess)
    return e;
  if (g.d == 128) {
    if (masked) sparse_attn_kernel<128, true, 0><<<grid, kThreads, smem, st>>>(mq, mk, mv, a);
    else if (raster) sparse_attn_kernel<128, false, 1><<<grid, kThreads, smem, st>>>(mq, mk, mv, a);
    else if (raster_out) sparse_attn_kernel<128, false, 2><<<grid, kThreads, smem, st>>>(mq, mk, mv, a);
    else sparse_attn_kernel<128, false, 0><<<grid, kThreads, smem, st>>>(mq, mk, mv, a);
  } else {
    if (masked) sparse_attn_kernel<64, true, 0><<<grid, kThreads, smem, st>>>(mq, mk, mv, a);
    else if (raster) sparse_attn_kernel<64, false, 1><<<grid, kThreads, smem, st>>>(mq, mk, mv, a);
    else if (raster_out) sparse_attn_kernel<64, false, 2><<<grid, kThreads, smem, st>>>(mq, mk, mv, a);
    else sparse_attn_kernel<64, false, 0><<<grid, kThreads, smem, st>>>(mq, mk, mv, a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    // report what the kernel needs next to what the launch asked for
    static thread_local char msg[256];
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, fn);
    snprintf(msg, sizeof msg,
             "sparse attention launch: %s (threads %d, regs/thread %d, max threads/block %d, "
             "static smem %zu, dynamic smem %d)",
             cudaGetErrorString(e), kThreads, fa.numRegs, fa.maxThreadsPerBlock,
             fa.sharedSizeBytes, smem);
    *why = msg;
  }
  return e;
}

}  // namespace vsa
