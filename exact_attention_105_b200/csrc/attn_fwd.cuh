// Forward kernel: O = softmax(Q K^T * scale [causal]) V and lse, on tcgen05
// tensor cores. A persistent kernel: one CTA per SM walks a fixed list of
// query blocks of 256 rows (two 128-row tiles) and overlaps the end of one
// block with the start of the next.
//
// Method: hysenlabs.com "FlashAttention: exakte Attention-Kernel fuer CUDA
// und ROCm", section "Die Schnittstellen von flash_attn_func bis KV-Cache",
// gives the formula. unite.ai "Was ist FlashAttention?", five-stage map:
//   stage 1: Q, K and V are cut into 128-row tiles;
//   stage 2: TMA brings each tile into shared memory (a ring of slots);
//   stage 3: S = Q K^T is computed per tile into tensor memory, then a
//            running row max / row sum normalises it (online softmax);
//   stage 4: O += P V accumulates in tensor memory, so the N x N matrix is
//            never materialised;
//   stage 5: the work is ordered for the B200: each CTA takes blocks from a
//            list, heaviest causal blocks first, and the next block's Q and
//            first K tile are loaded while the current block finishes.
//
// CTA layout (384 threads, 12 warps):
//   warps 0-3  softmax warpgroup for query tile 0 (rows 0..127 of the block)
//   warps 4-7  softmax warpgroup for query tile 1 (rows 128..255)
//   warp 8     TMA producer (one elected lane)
//   warp 9     TMEM allocator and MMA issuer (one elected lane)
//   warp 10    output store: TMA stores of the staged O tiles (one lane)
//   warp 11    idle
// Thread r of a softmax warpgroup owns TMEM lane r, i.e. query row r of its
// tile. That is the 32x32b access pattern: warp w%4 reads lanes 32*(w%4)...
//
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   [  0,128) S0 fp32; P0 (bf16 pairs) overwrites S0 columns [64,128)
//   [128,256) S1 fp32; P1 overwrites S1 columns [64,128)
//   [256,256+D) O0 fp32 accumulator, [384,384+D) O1 fp32 accumulator
// P_t(j) is read by the PV MMA, and the next S_t MMA overwrites the same
// columns. Both MMAs come from the same issuing thread, in that order, and
// the tensor pipe executes one thread's MMAs in issue order. The first PV of
// a block overwrites O_t only after that tile's epilogue of the previous
// block has read it (o_empty).
// One-tile blocks (problems too small to fill the SMs with two-tile blocks)
// run a double-buffered variant: S(j) of the one tile alternates between
// columns [0, 128) and [128, 256), and S(j + 2) is issued right after PV(j),
// so the softmax never waits for its own PV and next S. Its O rescale then
// first waits for PV(j - 1) (pv_done). The producer loads each K one key tile
// ahead of its V, so that with a 3-slot ring K(j + 2) is in place by then.
//
// Shared memory: two sets of Q tiles (the block being computed and the next
// one), then a ring of NS K/V slots. K_j and V_j take turns: K0, V0, K1, V1,
// ... The ring continues from one block to the next. Each 128 x D tile is
// stored as D/64 column blocks of 128 rows x 128 bytes, 128-byte swizzled,
// exactly as the TMA writes it. That is the canonical K-major SW128 layout for
// Q and K and the MN-major SW128 layout for V. At the end of a block, tile
// t's bf16 O is staged in its own Q slot, which no MMA reads any more, and
// the store warp writes it with a TMA store; the slot set is then free for
// the block after next.
#pragma once

#include "geometry.cuh"
#include "sm100.cuh"
#include "visibility.cuh"

namespace attn {

template <int D>
struct FwdCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kTileBytes = 128 * D * 2;          // one 128 x D bf16 tile
  static constexpr int kStages = (D == 128) ? 3 : 6;      // K/V ring slots
  static constexpr int kQOff = 0;                         // Q set s, tile t: (2 s + t) tiles in
  static constexpr int kKVOff = 4 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  // q_full[2] q_empty[2] kv_full[S] kv_empty[S] s_full[2] p_full[2] p_half[2]
  // o_full[2] o_empty[2] stage_full[4] mma_done[1] pv_done[1]
  static constexpr int kNumBars = 2 + 2 + 2 * kStages + 2 + 2 + 2 + 2 + 2 + 4 + 1 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;         // slack for 1024-B alignment
  static constexpr int kThreads = 384;
  static constexpr uint32_t kTxBytes = kTileBytes;
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
};

// Wait-site ids reported in the status word when a wait times out.
enum FwdSite : int {
  kSiteQFull = 1, kSiteKVFull = 2, kSiteKVEmpty = 3, kSiteSFull = 4, kSitePFull = 5,
  kSiteOFull = 6, kSiteQEmpty = 7, kSiteOEmpty = 8, kSiteStage = 9, kSitePHalf = 10,
  kSitePVDone = 11
};

// Register split: launched at kFwdRegsLaunch per thread (384 threads fill the
// 64K register file); warpgroup 2 (producer, MMA, store, idle) drops to
// kFwdRegsSmall and the two softmax warpgroups grow to kFwdRegsSoftmax.
// 2 * 216 + 72 = 3 * 168. The host refuses to launch if ptxas allocated a
// different launch count, since the grow would otherwise never be granted.
constexpr int kFwdRegsLaunch = 168;
constexpr int kFwdRegsSoftmax = 216;
constexpr int kFwdRegsSmall = 72;
static_assert(2 * kFwdRegsSoftmax + kFwdRegsSmall <= 3 * kFwdRegsLaunch, "register split");

// The list of work items. One item is a query block: rows [m0, m0 + rb) of
// one (batch, query head), rb = 256 (two tiles) or 128 (one tile, when two-tile
// blocks would leave SMs idle). Heads are taken in groups of `hg` (see the
// host), blocks from the last (heaviest when causal) to the first within a
// group, all heads of the group per block. Without a plan (below), CTA c of
// G takes list entries t G + c for even t and t G + G - 1 - c for odd t (a
// snake), which evens out the work of the CTAs over the heavy-to-light order
// when the blocks cost the same or the list is a whole number of snake periods.
struct FwdSched {
  int BH;            // batch * query heads
  int nmb;           // query blocks per head (of the longest sequence)
  int hg;            // heads per group
  int one_tile;      // 1: blocks of 128 rows (tile 1 never used)
  long long total;   // BH * nmb (the host keeps it below 2^31)
};

// A static plan of which CTA takes which list entries, for problems whose
// blocks differ in cost (causal). CTA c takes entries item[start[c]] ..
// item[start[c + 1] - 1] in that order. The host fills it by list
// scheduling: entries in list order, each to the CTA with the least work so
// far (key-tile steps plus a fixed cost per block). It travels in the kernel
// parameters, so a launch (or a CUDA graph that captured one) needs no device
// memory for it.
constexpr int kFwdPlanCtas = 160;
constexpr int kFwdPlanItems = 15360;
struct FwdPlan {
  uint16_t start[kFwdPlanCtas + 1];
  uint16_t item[kFwdPlanItems];
};
struct FwdNoPlan {
  int unused;
};
template <bool P>
struct FwdPlanArg {
  using type = FwdNoPlan;
};
template <>
struct FwdPlanArg<true> {
  using type = FwdPlan;
};

struct FwdBlock {
  SeqSpan sp;        // the sequence's rows (packed) or the fixed lengths
  int m0;            // first query row of tile 0
  int zq, zkv;       // TMA z coordinates of the query head and of its KV head
  int lo0, hi0, lo1, hi1;   // per tile: visible key tiles [lo, hi] (hi < lo: none)
  int jb, n_span;    // the block's key-tile stream jb .. jb + n_span - 1
  bool present;      // the block has rows (false: past a packed sequence's end)
  bool has1;         // tile 1 has rows
};

// List entry t of this CTA, or false when the list is exhausted.
template <int MODE, bool PACKED, bool PLAN>
__device__ __forceinline__ bool fwd_block(int t, const FwdSched& sc,
                                          const typename FwdPlanArg<PLAN>::type& plan, int Hq,
                                          int group, const SeqGeom& geom, KeyWindow win,
                                          FwdBlock& bk) {
  uint32_t idx;
  if constexpr (PLAN) {
    const int s0 = plan.start[blockIdx.x];
    if (t >= plan.start[blockIdx.x + 1] - s0) return false;
    idx = plan.item[s0 + t];
  } else {
    // 32-bit arithmetic: the host keeps the list below 2^31 entries, and
    // t G + G stays below 2^32 while t G < total.
    const uint32_t G = gridDim.x, c = blockIdx.x;
    idx = static_cast<uint32_t>(t) * G + ((t & 1) ? (G - 1 - c) : c);
    if (idx >= static_cast<uint32_t>(sc.total)) return false;
  }
  const uint32_t per_group = static_cast<uint32_t>(sc.hg) * static_cast<uint32_t>(sc.nmb);
  const uint32_t g = idx / per_group;
  const uint32_t r = idx - g * per_group;
  const int g0 = static_cast<int>(g) * sc.hg;
  const uint32_t gs = static_cast<uint32_t>(min(sc.hg, sc.BH - g0));
  const uint32_t mbi = r / gs;
  const int bh = g0 + static_cast<int>(r - mbi * gs);
  const int mb = sc.nmb - 1 - static_cast<int>(mbi);
  const int b = bh / Hq;
  const int hq = bh - b * Hq;
  bk.sp = seq_span<PACKED>(geom, b);
  bk.m0 = mb * (sc.one_tile ? 128 : 256);
  bk.present = bk.m0 < bk.sp.nq;
  bk.has1 = !sc.one_tile && bk.m0 + 128 < bk.sp.nq;
  bk.zq = PACKED ? hq : bh;
  bk.zkv = PACKED ? hq / group : b * (Hq / group) + hq / group;
  bk.lo0 = 0; bk.hi0 = -1; bk.lo1 = 0; bk.hi1 = -1;
  bk.jb = 0;
  bk.n_span = 0;
  if (bk.present) {
    win.off = bk.sp.nk - bk.sp.nq;                 // bottom-right alignment per sequence
    kv_tile_range<MODE>(bk.m0, min(bk.m0 + 127, bk.sp.nq - 1), bk.sp.nk, win, bk.lo0, bk.hi0);
    if (bk.has1)
      kv_tile_range<MODE>(bk.m0 + 128, min(bk.m0 + 255, bk.sp.nq - 1), bk.sp.nk, win, bk.lo1,
                          bk.hi1);
    const bool a0 = bk.hi0 >= bk.lo0, a1 = bk.hi1 >= bk.lo1;
    if (a0 || a1) {
      bk.jb = a0 ? bk.lo0 : bk.lo1;
      const int je = a1 ? bk.hi1 : bk.hi0;
      bk.n_span = je - bk.jb + 1;
    }
  }
  return true;
}

template <int D, int MODE, int FEAT, bool PLAN, bool DB>
__global__ void __launch_bounds__(384, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
           __nv_bfloat16* __restrict__ out,
           float* __restrict__ lse_out, int Hq, int group, SeqGeom geom, float scale_log2,
           KeyWindow win, Softcap cap, FwdSched sched,
           const __grid_constant__ typename FwdPlanArg<PLAN>::type plan) {
  constexpr bool SOFTCAP = (FEAT & kFeatSoftcap) != 0;
  constexpr bool PACKED = (FEAT & kFeatPacked) != 0;
  static_assert(FEAT == 0 || MODE == kMaskGeneral, "features run in the general mode");
  static_assert(!DB || !PLAN, "double-buffered S: one-tile blocks, no plan");
  using C = FwdCfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;                // per Q set: the block's Q tiles have landed
  uint64_t* q_empty = q_full + 2;         // per Q set: the block's O tiles have been stored
  uint64_t* kv_full = q_empty + 2;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;       // per tile
  uint64_t* p_full = s_full + 2;          // per tile: all of P is in TMEM
  uint64_t* p_half = p_full + 2;          // per tile: P of keys 0..63 is in TMEM
  uint64_t* o_full = p_half + 2;          // per tile: the block's last PV is done
  uint64_t* o_empty = o_full + 2;         // per tile: the epilogue has read O
  uint64_t* stage_full = o_empty + 2;     // per (Q set, tile): O staged or written directly
  uint64_t* mma_done = stage_full + 4;
  uint64_t* pv_done = mma_done + 1;       // double-buffered mode: a block's PV (not its last) done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&p_half[i], 128);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&stage_full[i], 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(pv_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Set-up done; the previous kernel's results must be visible from here on.
  grid_dep_wait();

  if (warp >= 8) {
    regs_shrink<kFwdRegsSmall>();
    if (warp == 8 && lane == 0) {
      // ---------------------------------------------------------- producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      uint32_t ld = 0;          // ring loads issued
      int k = 0;                // present blocks so far (Q set k % 2)
      int last_q0 = -1, last_q1 = -1;   // block index of the last Q load per set
      bool ok = true;
      FwdBlock bk;
      for (int t = 0; ok && fwd_block<MODE, PACKED, PLAN>(t, sched, plan, Hq, group, geom, win, bk); ++t) {
        if (!bk.present) continue;
        const int set = k & 1;
        if (k >= 2 && !mbar_wait(&q_empty[set], ((k >> 1) - 1) & 1, abort_flag, kSiteQEmpty)) {
          ok = false;
          break;
        }
        const int ntiles = bk.has1 ? 2 : 1;
        mbar_expect_tx(&q_full[set], ntiles * C::kTxBytes);
        for (int tt = 0; tt < ntiles; ++tt) {
#pragma unroll
          for (int a = 0; a < D / 64; ++a)
            tma_load_3d(smem + C::kQOff + (2 * set + tt) * C::kTileBytes + a * 16384, &tm_q,
                        &q_full[set], a * 64, bk.sp.q0 + bk.m0 + tt * 128, bk.zq);
        }
        if (set) last_q1 = k; else last_q0 = k;
        if constexpr (DB) {
          // Next ring load: K (w = 0) or V (w = 1) of key tile j.
          auto load = [&](int w, int j) {
            const uint32_t s = ld % NS;
            if (ld >= static_cast<uint32_t>(NS) &&
                !mbar_wait(&kv_empty[s], (ld / NS - 1) & 1u, abort_flag, kSiteKVEmpty))
              return false;
            mbar_expect_tx(&kv_full[s], C::kTxBytes);
#pragma unroll
            for (int a = 0; a < D / 64; ++a)
              tma_load_3d(smem + C::kKVOff + s * C::kTileBytes + a * 16384, w ? &tm_v : &tm_k,
                          &kv_full[s], a * 64, bk.sp.k0 + j * 128, bk.zkv);
            ++ld;
            return true;
          };
          // With a 3-slot ring, K runs one key tile ahead: K_0, then K_m,
          // V_(m-1) for m = 1 .. n-1, then V_(n-1), so that K_(j+2) can land
          // during the softmax of S(j). Deeper rings keep the plain order
          // (measured 3 % faster at d = 64).
          const int n = bk.n_span;
          if (NS < 4) {
            for (int m = 0; ok && m <= n; ++m) {
              if (m < n && !load(0, bk.jb + m)) ok = false;
              if (ok && m > 0 && !load(1, bk.jb + m - 1)) ok = false;
            }
          } else {
            for (int m = 0; ok && m < n; ++m)
              if (!load(0, bk.jb + m) || !load(1, bk.jb + m)) ok = false;
          }
        } else {
          for (int j = bk.jb; ok && j < bk.jb + bk.n_span; ++j) {
            for (int w = 0; w < 2; ++w) {
              const uint32_t s = ld % NS;
              if (ld >= static_cast<uint32_t>(NS) &&
                  !mbar_wait(&kv_empty[s], (ld / NS - 1) & 1u, abort_flag, kSiteKVEmpty)) {
                ok = false;
                break;
              }
              mbar_expect_tx(&kv_full[s], C::kTxBytes);
#pragma unroll
              for (int a = 0; a < D / 64; ++a)
                tma_load_3d(smem + C::kKVOff + s * C::kTileBytes + a * 16384, w ? &tm_v : &tm_k,
                            &kv_full[s], a * 64, bk.sp.k0 + j * 128, bk.zkv);
              ++ld;
            }
          }
        }
        ++k;
      }
      // Let every copy this thread started land before the CTA can exit.
      if (last_q0 >= 0) mbar_wait_drain(&q_full[0], (last_q0 >> 1) & 1);
      if (last_q1 >= 0) mbar_wait_drain(&q_full[1], (last_q1 >> 1) & 1);
      const uint32_t first = ld > static_cast<uint32_t>(NS) ? ld - NS : 0u;
      for (uint32_t i = first; i < ld; ++i) mbar_wait_drain(&kv_full[i % NS], (i / NS) & 1u);
    } else if (warp == 9 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);
      auto issue_qk = [&](int t, int set, uint32_t slot) {
        const SDesc qd =
            sdesc_sw128_split(sbase + C::kQOff + (2 * set + t) * C::kTileBytes, 16, 1024);
        const SDesc kd = sdesc_sw128_split(sbase + C::kKVOff + slot * C::kTileBytes, 16, 1024);
        mma_ss_w<0>(tmem + t * 128, qd.lo, qd.hi, kd.lo, kd.hi, kIdescQK);
#pragma unroll
        for (int kk = 1; kk < D / 16; ++kk) {
          const uint32_t o = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          mma_ss_w<1>(tmem + t * 128, qd.lo + o, qd.hi, kd.lo + o, kd.hi, kIdescQK);
        }
      };
      // O_t += P (keys [64 h, 64 h + 64)) V. P is packed bf16 in TMEM columns
      // [64, 128) of the tile's S region, 32 columns per half.
      auto issue_pv_half = [&](int t, uint32_t slot, int h, bool acc) {
        const SDesc vd = sdesc_sw128_split(sbase + C::kKVOff + slot * C::kTileBytes, 16384, 1024);
        const uint32_t pa = tmem + t * 128 + 64 + 32 * h, od = tmem + 256 + t * 128;
        mma_ts_w<-1>(od, pa, vd.lo + 4 * h * 128, vd.hi, kIdescPV, acc ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 4; ++kk)
          mma_ts_w<1>(od, pa + kk * 8, vd.lo + (4 * h + kk) * 128, vd.hi, kIdescPV);
      };
      auto kv_wait = [&](uint32_t idx) {
        return mbar_wait(&kv_full[idx % NS], (idx / NS) & 1u, abort_flag, kSiteKVFull);
      };

      bool ok = true, any = false;
      uint32_t base = 0;                  // ring index of the block's first load
      int k = 0;                          // present blocks
      // Per tile: P hand-overs consumed, blocks accumulated (scalars, never a
      // runtime-indexed array: that would live in local memory).
      uint32_t pc0 = 0, pc1 = 0;
      int oc0 = 0, oc1 = 0;
      FwdBlock bk;
      if constexpr (DB) {
        // One-tile blocks with S double-buffered in TMEM columns [0, 128) and
        // [128, 256) (the second tile's, unused here): S(j + 2) is issued right
        // after PV(j), so the softmax finds S(j + 1) ready when it finishes
        // S(j) instead of waiting for PV(j) and S(j + 1) in turn.
        auto issue_qk_db = [&](uint32_t b, int set, uint32_t slot) {
          const SDesc qd =
              sdesc_sw128_split(sbase + C::kQOff + 2 * set * C::kTileBytes, 16, 1024);
          const SDesc kd = sdesc_sw128_split(sbase + C::kKVOff + slot * C::kTileBytes, 16, 1024);
          mma_ss_w<0>(tmem + b * 128, qd.lo, qd.hi, kd.lo, kd.hi, kIdescQK);
#pragma unroll
          for (int kk = 1; kk < D / 16; ++kk) {
            const uint32_t o = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
            mma_ss_w<1>(tmem + b * 128, qd.lo + o, qd.hi, kd.lo + o, kd.hi, kIdescQK);
          }
        };
        auto issue_pv_db = [&](uint32_t b, uint32_t slot, int h, bool acc) {
          const SDesc vd =
              sdesc_sw128_split(sbase + C::kKVOff + slot * C::kTileBytes, 16384, 1024);
          const uint32_t pa = tmem + b * 128 + 64 + 32 * h, od = tmem + 256;
          mma_ts_w<-1>(od, pa, vd.lo + 4 * h * 128, vd.hi, kIdescPV, acc ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < 4; ++kk)
            mma_ts_w<1>(od, pa + kk * 8, vd.lo + (4 * h + kk) * 128, vd.hi, kIdescPV);
        };
        for (int t = 0; ok && fwd_block<MODE, PACKED, PLAN>(t, sched, plan, Hq, group, geom, win, bk);
             ++t) {
          if (!bk.present) continue;
          const int set = k & 1;
          if (!mbar_wait(&q_full[set], (k >> 1) & 1, abort_flag, kSiteQFull)) { ok = false; break; }
          ++k;
          const int n = bk.n_span;        // the one tile's key tiles are the block's span
          if (n == 0) continue;
          any = true;
          // Ring positions in the producer's order, from the block's first
          // load. 3-slot ring (K one key tile ahead): K_m at 2m - 1 (K_0 at
          // 0), V_m at 2m + 2 (the last V at 2n - 1). Deeper rings: K_m at
          // 2m, V_m at 2m + 1.
          auto pos_k = [&](int m) {
            return base + (NS >= 4 ? 2u * m : (m == 0 ? 0u : 2u * m - 1u));
          };
          auto pos_v = [&](int m) {
            return base + (NS >= 4 ? 2u * m + 1u : (m == n - 1 ? 2u * n - 1u : 2u * m + 2u));
          };
          for (int jj = 0; ok && jj < 2 && jj < n; ++jj) {
            if (!kv_wait(pos_k(jj))) { ok = false; break; }
            tc_fence_after();
            issue_qk_db(jj, set, pos_k(jj) % NS);
            tc_commit(&s_full[jj]);
            tc_commit(&kv_empty[pos_k(jj) % NS]);
          }
          for (int jj = 0; ok && jj < n; ++jj) {
            const uint32_t b = jj & 1, iv = pos_v(jj);
            if (!kv_wait(iv) || !mbar_wait(&p_half[0], pc0 & 1u, abort_flag, kSitePHalf)) {
              ok = false;
              break;
            }
            if (jj == 0 && oc0 > 0 &&
                !mbar_wait(&o_empty[0], (oc0 - 1) & 1, abort_flag, kSiteOEmpty)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv_db(b, iv % NS, 0, jj > 0);
            if (!mbar_wait(&p_full[0], pc0 & 1u, abort_flag, kSitePFull)) { ok = false; break; }
            ++pc0;
            tc_fence_after();
            issue_pv_db(b, iv % NS, 1, true);
            if (jj == n - 1) {
              tc_commit(&o_full[0]);
              ++oc0;
            } else {
              tc_commit(pv_done);
            }
            tc_commit(&kv_empty[iv % NS]);
            if (jj + 2 < n) {
              // Into the buffer PV(jj) has just read: the pipe runs this
              // thread's MMAs in issue order.
              const uint32_t ik = pos_k(jj + 2);
              if (!kv_wait(ik)) { ok = false; break; }
              tc_fence_after();
              issue_qk_db(b, set, ik % NS);
              tc_commit(&s_full[b]);
              tc_commit(&kv_empty[ik % NS]);
            }
          }
          base += 2 * n;
        }
      } else {
        for (int t = 0; ok && fwd_block<MODE, PACKED, PLAN>(t, sched, plan, Hq, group, geom, win, bk); ++t) {
          if (!bk.present) continue;
          const int set = k & 1;
          if (!mbar_wait(&q_full[set], (k >> 1) & 1, abort_flag, kSiteQFull)) { ok = false; break; }
          ++k;
          if (bk.n_span == 0) continue;
          any = true;
          const int jb = bk.jb, je = bk.jb + bk.n_span;
          auto lo_t = [&](int tt) { return tt ? bk.lo1 : bk.lo0; };
          auto hi_t = [&](int tt) { return tt ? bk.hi1 : bk.hi0; };
          // Ring positions: K_j at base + 2 (j - jb), V_j at base + 2 (j - jb) + 1.
          if (!kv_wait(base)) { ok = false; break; }
          tc_fence_after();
  #pragma unroll
          for (int tt = 0; tt < 2; ++tt)
            if (hi_t(tt) >= lo_t(tt) && lo_t(tt) == jb) {
              issue_qk(tt, set, base % NS);
              tc_commit(&s_full[tt]);
            }
          tc_commit(&kv_empty[base % NS]);
          for (int j = jb; ok && j < je; ++j) {
            const uint32_t iv = base + 2 * (j - jb) + 1, ik = iv + 1;
            if (!kv_wait(iv)) { ok = false; break; }
            tc_fence_after();
            bool k_ready = false;
            auto need_k_next = [&]() {
              if (!k_ready) {
                if (!kv_wait(ik)) return false;
                tc_fence_after();
                k_ready = true;
              }
              return true;
            };
  #pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
              const int lo = lo_t(tt), hi = hi_t(tt);
              if (hi < lo) continue;
              if (j >= lo && j <= hi) {
                uint32_t& pc = tt ? pc1 : pc0;
                int& oc = tt ? oc1 : oc0;
                // P arrives in two halves: the first half's PV runs while the
                // softmax still computes the second half. The next S tile
                // overwrites P, so it follows the second half's PV.
                if (!mbar_wait(&p_half[tt], pc & 1u, abort_flag, kSitePHalf)) { ok = false; break; }
                // The first accumulation of a block overwrites O_t: the previous
                // block's epilogue must have read it.
                if (j == lo && oc > 0 &&
                    !mbar_wait(&o_empty[tt], (oc - 1) & 1, abort_flag, kSiteOEmpty)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                issue_pv_half(tt, iv % NS, 0, j > lo);
                if (!mbar_wait(&p_full[tt], pc & 1u, abort_flag, kSitePFull)) { ok = false; break; }
                ++pc;
                tc_fence_after();
                issue_pv_half(tt, iv % NS, 1, true);
                if (j == hi) {
                  tc_commit(&o_full[tt]);
                  ++oc;
                } else {
                  if (!need_k_next()) { ok = false; break; }
                  issue_qk(tt, set, ik % NS);
                  tc_commit(&s_full[tt]);
                }
              } else if (lo == j + 1) {
                // This tile's first key tile is the next one.
                if (!need_k_next()) { ok = false; break; }
                issue_qk(tt, set, ik % NS);
                tc_commit(&s_full[tt]);
              }
            }
            // K_{j+1} feeds some tile whenever j + 1 is in the span (the two
            // tiles' ranges overlap or touch); release its slot even if no tile
            // used it.
            if (ok && j + 1 < je && !need_k_next()) ok = false;
            if (!ok) break;
            tc_commit(&kv_empty[iv % NS]);
            if (k_ready) tc_commit(&kv_empty[ik % NS]);
          }
          base += 2 * bk.n_span;
        }
      }
      // Let this thread's MMAs finish before TMEM can be released.
      if (any) {
        tc_commit(mma_done);
        mbar_wait_drain(mma_done, 0);
      }
    } else if (warp == 10 && lane == 0) {
      // ---------------------------------------------------------- output store
      tma_prefetch_desc(&tm_o);
      int k = 0;
      FwdBlock bk;
      for (int t = 0; fwd_block<MODE, PACKED, PLAN>(t, sched, plan, Hq, group, geom, win, bk); ++t) {
        if (!bk.present) continue;
        const int set = k & 1;
        bool ok = true;
        for (int tt = 0; tt < 2 && ok; ++tt) {
          if (!mbar_wait(&stage_full[2 * set + tt], (k >> 1) & 1, abort_flag, kSiteStage)) {
            ok = false;
            break;
          }
          const int r_first = bk.m0 + tt * 128;
          const bool rows = tt == 0 || bk.has1;
          const bool tma_tile = rows && (!PACKED || r_first + 128 <= bk.sp.nq);
          if (tma_tile) {
            uint8_t* tile = smem + C::kQOff + (2 * set + tt) * C::kTileBytes;
#pragma unroll
            for (int a = 0; a < D / 64; ++a)
              tma_store_3d(&tm_o, tile + a * 16384, a * 64, bk.sp.q0 + r_first, bk.zq);
            bulk_commit_group();
          }
        }
        if (!ok) break;
        bulk_wait_read_all();
        mbar_arrive(&q_empty[set]);
        ++k;
      }
      bulk_wait_read_all();
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    regs_grow<kFwdRegsSoftmax>();
    const int t = warp >> 2;
    const int quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t t_s = tmem + lane_base + t * 128;
    const uint32_t t_o = tmem + lane_base + 256 + t * 128;
    const int tr = quad * 32 + lane;                       // row within the tile
    uint32_t sc = 0;          // S hand-overs consumed by this tile
    uint32_t sc1 = 0;         // double-buffered mode: those of the second buffer
    uint32_t pvc = 0;         // double-buffered mode: PV completions waited for
    int oc = 0;               // blocks whose O this tile accumulated
    int k = 0;                // present blocks
    bool ok = true;
    FwdBlock bk;
    for (int it = 0; fwd_block<MODE, PACKED, PLAN>(it, sched, plan, Hq, group, geom, win, bk); ++it) {
      if (!bk.present) continue;
      const int set = k & 1;
      ++k;
      const int Nq = bk.sp.nq, Nk = bk.sp.nk;
      const int r_first = bk.m0 + t * 128;                 // first and last row of this tile
      const bool rows = t == 0 || bk.has1;
      const int r_last = min(r_first + 127, Nq - 1);
      const int row = r_first + tr;
      const int lo = t ? bk.lo1 : bk.lo0, hi = t ? bk.hi1 : bk.hi0;
      const int n = rows ? max(0, hi - lo + 1) : 0;
      win.off = Nk - Nq;
      // Visible keys of this row: [k_lo, k_hi] (k_hi < k_lo: none).
      const int k_lo = (MODE == kMaskGeneral) ? max(0, win.lo(row)) : 0;
      const int k_hi = (MODE == kMaskGeneral)
                           ? min(Nk - 1, win.hi(row))
                           : ((MODE == kMaskCausal) ? min(row, Nk - 1) : Nk - 1);
      const int nkv = (Nk + 127) >> 7;
      const bool ragged = (Nk & 127) != 0;
      // What the epilogue needs of the block, computed now so that the block
      // record is dead during the key loop (register pressure).
      const bool row_ok = rows && row < Nq;
      const bool tma_tile = rows && (!PACKED || r_first + 128 <= Nq);
      float* lse_dst =
          lse_out + bk.zq * (PACKED ? geom.lse_z : static_cast<long long>(Nq)) + bk.sp.q0 + row;
      __nv_bfloat16* o_dst =
          out + bk.zq * (PACKED ? geom.o_z : static_cast<long long>(Nq) * D) +
          (bk.sp.q0 + row) * (PACKED ? geom.o_row : static_cast<long long>(D));

      float m_run = -INFINITY;   // running max, log2 units (scaled logits * log2 e)
      float l_run = 0.f;         // running sum of 2^(t - m_run), unrounded (for lse)
      float l_mma = 0.f;         // running sum of the bf16-rounded P fed to the MMA (for O)
      for (int jj = 0; ok && jj < n; ++jj) {
        const int j = lo + jj;                             // key tile
        const int kb = j * 128;
        // Double-buffered mode: odd steps use the second S buffer and barrier.
        const bool odd = DB && (jj & 1);
        const uint32_t t_sb = odd ? t_s + 128 : t_s;
        if (!mbar_wait(&s_full[odd ? 1 : t], (odd ? sc1 : sc) & 1u, abort_flag, kSiteSFull)) {
          ok = false;
          break;
        }
        if (odd) ++sc1; else ++sc;
        tc_fence_after();
        uint32_t r0[32], r1[32], r2[32], r3[32];
        tmem_ld32(t_sb + 0, r0);
        tmem_ld32(t_sb + 32, r1);
        tmem_ld32(t_sb + 64, r2);
        tmem_ld32(t_sb + 96, r3);
        tmem_ld_wait(r0);
        reg_fence(r1);
        reg_fence(r2);
        reg_fence(r3);

        if constexpr (SOFTCAP) {
          // Scores become capped logits in log2 units, in place. The mask below
          // then sets -inf on the capped values.
          auto cap_block = [&](uint32_t (&rr)[32]) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              rr[e] = f2u(cap.out * softcap_tanh(u2f(rr[e]), cap));
          };
          cap_block(r0);
          cap_block(r1);
          cap_block(r2);
          cap_block(r3);
        }
        // Only tiles that straddle an edge of some row's visible range are masked.
        bool edge;
        if (MODE == kMaskNone) edge = ragged && j == nkv - 1;
        else if (MODE == kMaskCausal) edge = jj == n - 1;
        else edge = kb < win.lo(r_last) || kb + 127 > min(Nk - 1, win.hi(r_first));
        if (edge) {
          const int c_lo = k_lo - kb, c_hi = k_hi - kb;     // keep columns [c_lo, c_hi]
          const uint32_t ninf = f2u(-INFINITY);
          if (MODE == kMaskGeneral) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (e < c_lo || e > c_hi) r0[e] = ninf;
              if (32 + e < c_lo || 32 + e > c_hi) r1[e] = ninf;
              if (64 + e < c_lo || 64 + e > c_hi) r2[e] = ninf;
              if (96 + e < c_lo || 96 + e > c_hi) r3[e] = ninf;
            }
          } else {                                          // k_lo = 0: one-sided
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (e > c_hi) r0[e] = ninf;
              if (32 + e > c_hi) r1[e] = ninf;
              if (64 + e > c_hi) r2[e] = ninf;
              if (96 + e > c_hi) r3[e] = ninf;
            }
          }
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          mx0 = fmax3f(mx0, u2f(r0[e]), u2f(r0[e + 1]));
          mx1 = fmax3f(mx1, u2f(r1[e]), u2f(r1[e + 1]));
          mx2 = fmax3f(mx2, u2f(r2[e]), u2f(r2[e + 1]));
          mx3 = fmax3f(mx3, u2f(r3[e]), u2f(r3[e + 1]));
        }
        // (Capped logits are already scaled to log2 units.)
        const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * (SOFTCAP ? 1.0f : scale_log2);
        const float m_new = fmaxf(m_run, m_tile);
        // Lazy rescale: keep the stale max unless the new one is more than 2^8 larger.
        const bool need = m_new > m_run + 8.0f;
        if constexpr (DB) {
          // S(jj) was issued before PV(jj - 1), which may still be adding to O.
          if (jj > 0) {
            if (!mbar_wait(pv_done, pvc & 1u, abort_flag, kSitePVDone)) { ok = false; break; }
            ++pvc;
            tc_fence_after();
          }
        }
        if (jj > 0 && __any_sync(0xffffffffu, need)) {
          const float f = need ? fast_exp2(m_run - m_new) : 1.0f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_o + c * 32, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = f2u(u2f(o[e]) * f);
            tmem_st32(t_o + c * 32, o);
          }
        }
        if (need) {
          const float f = fast_exp2(m_run - m_new);
          l_run *= f;
          l_mma *= f;
          m_run = m_new;
        }
        const float sl = SOFTCAP ? 1.0f : scale_log2;
        const float2 sc2 = make_float2(sl, sl);
        // A row with no visible key so far keeps m_run = -inf; its p are all 0.
        const float neg_m = (m_run == -INFINITY) ? 0.0f : -m_run;
        const float2 nm2 = make_float2(neg_m, neg_m);
        float2 ex0 = make_float2(0.f, 0.f), ex1 = make_float2(0.f, 0.f);
        float q0 = 0.f, q1 = 0.f, q2 = 0.f, q3 = 0.f;
        // The 128 scores become 64 packed bf16 pairs in registers, stored to
        // TMEM as two 32-column halves. The first half's store is waited for
        // only after the third chunk's exponentials, so its latency hides
        // behind them; a wait right after each 32-column chunk stalled every
        // chunk (measured 4 % slower on 16K-key rows). The S registers die as
        // the P words are produced, so the peak stays near 150 registers. Two
        // row sums are kept. The exact one (unrounded p, paired
        // fp32 adds) gives lse. The other adds the bf16-rounded p that the PV MMA
        // consumes, and O is divided by it, so O's weights sum to one as they do
        // in the definition (a one-hot row returns V exactly).
        uint32_t pall[64];
        auto emit = [&](const uint32_t (&rr)[32], uint32_t col) {
          uint32_t* pw = pall + col;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float2 x = ffma2(make_float2(u2f(rr[2 * e]), u2f(rr[2 * e + 1])), sc2, nm2);
            x.x = fast_exp2(x.x);
            x.y = fast_exp2(x.y);
            const uint32_t pk = pack_bf16x2(x.x, x.y);
            if (e & 1) {
              ex1 = fadd2(ex1, x);
              if (e & 2) q3 = add_bf16x2_to_f32(q3, pk); else q1 = add_bf16x2_to_f32(q1, pk);
            } else {
              ex0 = fadd2(ex0, x);
              if (e & 2) q2 = add_bf16x2_to_f32(q2, pk); else q0 = add_bf16x2_to_f32(q0, pk);
            }
            pw[e] = pk;
          }
        };
        // P of keys 0..63 goes to TMEM columns 64..95 of the S region and is
        // handed over first; keys 64..127 go to columns 96..127.
        emit(r0, 0);
        emit(r1, 16);
        tmem_st32(t_sb + 64, *reinterpret_cast<const uint32_t(*)[32]>(pall));
        emit(r2, 32);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_half[t]);
        emit(r3, 48);
        tmem_st32(t_sb + 96, *reinterpret_cast<const uint32_t(*)[32]>(pall + 32));
        const float2 ex = fadd2(ex0, ex1);
        l_run += ex.x + ex.y;
        l_mma += (q0 + q1) + (q2 + q3);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }

      // Epilogue. A row that saw no key (l = 0) gets O = 0 and lse = -inf.
      // The tile's O is staged in its own Q slot of this block's set: the
      // block's last S MMA of this tile finished before o_full. The block's
      // Q load is waited for by every warpgroup, keys or not: it follows the
      // slot's previous store (so zeros may be staged), and every q_full
      // phase is then observed in order, which keeps the parity test exact.
      const bool has_o = n > 0;
      if (ok) ok = mbar_wait(&q_full[set], ((k - 1) >> 1) & 1, abort_flag, kSiteQFull);
      if (ok && has_o) ok = mbar_wait(&o_full[t], oc & 1, abort_flag, kSiteOFull);
      if (has_o) ++oc;
      // Every thread of the warpgroup reaches this barrier once per block, so
      // a wait that gave up anywhere ends the loop for the whole warpgroup.
      if (!named_barrier_and(1 + t, 128, ok)) { ok = false; break; }
      if (rows) {
        const float inv_l = (l_mma > 0.f) ? 1.0f / l_mma : 0.f;
        if (has_o) tc_fence_after();
        uint8_t* tile = smem + C::kQOff + (2 * set + t) * C::kTileBytes;
        // All of the row's O columns are loaded before one wait (the S and P
        // registers are dead here), so the loads overlap.
        uint32_t oall[D / 32][32];
        if (has_o) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tmem_ld32(t_o + c * 32, oall[c]);
          tmem_ld_wait(oall[0]);
#pragma unroll
          for (int c = 1; c < D / 32; ++c) reg_fence(oall[c]);
        } else {
#pragma unroll
          for (int c = 0; c < D / 32; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) oall[c][e] = 0u;
        }
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          const uint32_t (&o)[32] = oall[c];
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(u2f(o[2 * e]) * inv_l, u2f(o[2 * e + 1]) * inv_l);
          if (tma_tile) {
            uint8_t* rowp = tile + (c >> 1) * 16384 + tr * 128;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const int ch = (c & 1) * 4 + qq;
              *reinterpret_cast<uint4*>(rowp + ((ch ^ (tr & 7)) << 4)) =
                  make_uint4(pk[4 * qq], pk[4 * qq + 1], pk[4 * qq + 2], pk[4 * qq + 3]);
            }
          } else if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(o_dst + c * 32);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
            dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
          }
        }
        if (row_ok)
          *lse_dst = (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
        tc_fence_before();
        if (tma_tile) fence_proxy_async_smem();
      }
      named_barrier_sync(1 + t, 128);
      if (quad == 0 && lane == 0) {
        if (has_o) mbar_arrive(&o_empty[t]);
        mbar_arrive(&stage_full[2 * set + t]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  grid_dep_launch();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
