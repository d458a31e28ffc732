// Forward kernel: O = softmax(Q K^T * scale [causal]) V and lse, one CTA per
// (batch*head, 256-row query block), on tcgen05 tensor cores.
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
//   stage 5: the grid is ordered for the B200: every head's heaviest causal
//            block first, lighter blocks after.
//
// CTA layout (384 threads, 12 warps):
//   warps 0-3  softmax warpgroup for query tile 0 (rows 0..127 of the block)
//   warps 4-7  softmax warpgroup for query tile 1 (rows 128..255)
//   warp 8     TMA producer (one elected lane)
//   warp 9     TMEM allocator and MMA issuer (one elected lane)
//   warps 10-11 idle
// Thread r of a softmax warpgroup owns TMEM lane r, i.e. query row r of its
// tile. That is the 32x32b access pattern: warp w%4 reads lanes 32*(w%4)...
//
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   [  0,128) S0 fp32; P0 (bf16 pairs) overwrites S0 columns [64,128)
//   [128,256) S1 fp32; P1 overwrites S1 columns [64,128)
//   [256,256+D) O0 fp32 accumulator, [384,384+D) O1 fp32 accumulator
// P_t(j) is read by the PV MMA, and the next S_t(j+1) MMA overwrites the
// same columns. Both MMAs come from the same issuing thread, in that order,
// and the tensor pipe executes one thread's MMAs in issue order.
//
// Shared memory: Q0, Q1 tiles, then a ring of NSTAGE K/V slots. K_j and V_j
// take turns: K0, V0, K1, V1, ... Each 128 x D tile is stored as D/64
// column blocks of 128 rows x 128 bytes, 128-byte swizzled, exactly as the
// TMA writes it. That is the canonical K-major SW128 layout for Q and K and
// the MN-major SW128 layout for V. At the end, tile t's bf16 O is staged in
// Q_t's slot in the same layout and written with a TMA store.
#pragma once

#include "geometry.cuh"
#include "sm100.cuh"
#include "visibility.cuh"

namespace attn {

template <int D>
struct FwdCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kTileBytes = 128 * D * 2;          // one 128 x D bf16 tile
  static constexpr int kStages = (D == 128) ? 4 : 6;      // K/V ring slots
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  // q_full[2] kv_full[S] kv_empty[S] s_full[2] p_full[2] o_full[2] mma_done[1]
  static constexpr int kNumBars = 2 + 2 * kStages + 2 + 2 + 2 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;         // slack for 1024-B alignment
  static constexpr int kThreads = 384;
  static constexpr uint32_t kTxBytes = kTileBytes;
};

// Wait-site ids reported in the status word when a wait times out.
enum FwdSite : int {
  kSiteQFull = 1, kSiteKVFull = 2, kSiteKVEmpty = 3, kSiteSFull = 4, kSitePFull = 5,
  kSiteOFull = 6
};

// Register split: launched at kFwdRegsLaunch per thread (384 threads fill the
// 64K register file); warpgroup 2 (producer, MMA, idle) drops to
// kFwdRegsSmall and the two softmax warpgroups grow to kFwdRegsSoftmax.
// 2 * 216 + 72 = 3 * 168. The host refuses to launch if ptxas allocated a
// different launch count, since the grow would otherwise never be granted.
constexpr int kFwdRegsLaunch = 168;
constexpr int kFwdRegsSoftmax = 216;
constexpr int kFwdRegsSmall = 72;
static_assert(2 * kFwdRegsSoftmax + kFwdRegsSmall <= 3 * kFwdRegsLaunch, "register split");

template <int D, int MODE, int FEAT>
__global__ void __launch_bounds__(384, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
           __nv_bfloat16* __restrict__ out,
           float* __restrict__ lse_out, int Hq, int group, SeqGeom geom, float scale_log2,
           KeyWindow win, Softcap cap, int one_tile, int hg) {
  constexpr bool SOFTCAP = (FEAT & kFeatSoftcap) != 0;
  constexpr bool PACKED = (FEAT & kFeatPacked) != 0;
  static_assert(FEAT == 0 || MODE == kMaskGeneral, "features run in the general mode");
  using C = FwdCfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* kv_full = q_full + 2;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* mma_done = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  const int warp = warp_id();
  const int lane = lane_id();
  // 1-D grid over (batch * query head, 256-row query block). The heads are
  // taken in groups of hg (all of them when hg covers every head); within a
  // group, (batch, query head) runs fastest and the blocks go from the last
  // (heaviest when causal) to the first. Causal problems use one group, so
  // every head's heaviest block is dispatched before any lighter one, which
  // keeps the tail short. Unmasked problems, whose blocks all cost the same,
  // use groups whose K and V fit in L2, so a group's blocks reread K/V from
  // L2 rather than DRAM.
  // Rows per CTA: two 128-row tiles, or one when the problem is too small to
  // fill the GPU with two-tile CTAs (more CTAs, one tile each).
  const int rb = one_tile ? 128 : 256;
  const int nmb = (geom.Nq + rb - 1) / rb;
  const int BH = gridDim.x / nmb;
  const int per_group = hg * nmb;
  const int grp = blockIdx.x / per_group;
  const int g0 = grp * hg;
  const int gs = min(hg, BH - g0);
  const int rr = blockIdx.x - grp * per_group;
  const int mbi = rr / gs;
  const int bh = g0 + (rr - mbi * gs);             // b * Hq + hq
  const int b = bh / Hq;
  const int hq = bh - b * Hq;
  const int mb = nmb - 1 - mbi;
  const SeqSpan sp = seq_span<PACKED>(geom, b);
  const int Nq = sp.nq, Nk = sp.nk;
  const int m0 = mb * rb;                          // first query row of this CTA
  if (m0 >= Nq) return;                            // packed batch: past this sequence's rows
  win.off = Nk - Nq;                               // bottom-right alignment per sequence
  // TMA z coordinates of the query head and its KV head (GQA: contiguous groups).
  const int zq = PACKED ? hq : bh;
  const int zkv = PACKED ? hq / group : b * (Hq / group) + hq / group;
  const int nkv = (Nk + 127) >> 7;

  // Per query tile t: KV tiles [lo_t(t), hi_t(t)] (n_t(t) of them). A tile whose
  // rows exist but see no key has n_t = 0 and writes O = 0, lse = -inf. The
  // CTA streams KV tiles jb..je, the union of its tiles' ranges. The bounds
  // are scalars with select accessors, never an array indexed by a runtime
  // tile number: that would live in local memory and be reloaded after every
  // barrier wait on the MMA issue path.
  int lo0 = 0, hi0 = -1, lo1 = 0, hi1 = -1;
  kv_tile_range<MODE>(m0, min(m0 + 127, Nq - 1), Nk, win, lo0, hi0);
  if (!one_tile && m0 + 128 < Nq)
    kv_tile_range<MODE>(m0 + 128, min(m0 + 255, Nq - 1), Nk, win, lo1, hi1);
  const int n0 = max(0, hi0 - lo0 + 1), n1 = max(0, hi1 - lo1 + 1);
  auto lo_t = [&](int t) { return t ? lo1 : lo0; };
  auto hi_t = [&](int t) { return t ? hi1 : hi0; };
  auto n_t = [&](int t) { return t ? n1 : n0; };
  const int jb = (n_t(0) > 0) ? lo_t(0) : lo_t(1);
  const int je = (n_t(1) > 0) ? hi_t(1) : hi_t(0);
  const int n_span = (n_t(0) > 0 || n_t(1) > 0) ? je - jb + 1 : 0;

  if (threadIdx.x == 0) {
    mbar_init(&q_full[0], 1);
    mbar_init(&q_full[1], 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_full[t], 1);
    }
    mbar_init(mma_done, 1);
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

  if (warp >= 8) {
    regs_shrink<kFwdRegsSmall>();
    if (warp == 8 && lane == 0) {
      // ---------------------------------------------------------- producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (n_t(t) > 0) {
          mbar_expect_tx(&q_full[t], C::kTxBytes);
#pragma unroll
          for (int a = 0; a < D / 64; ++a)
            tma_load_3d(smem + C::kQOff + t * C::kTileBytes + a * 16384, &tm_q, &q_full[t],
                        a * 64, sp.q0 + m0 + t * 128, zq);
        }
      }
      uint32_t issued = 0;
      bool ok = true;
      for (int j = jb; j < jb + n_span && ok; ++j) {
        for (int w = 0; w < 2; ++w) {
          const uint32_t s = issued % NS;
          const uint32_t round = issued / NS;
          if (round > 0 && !mbar_wait(&kv_empty[s], (round - 1) & 1u, abort_flag, kSiteKVEmpty)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&kv_full[s], C::kTxBytes);
#pragma unroll
          for (int a = 0; a < D / 64; ++a)
            tma_load_3d(smem + C::kKVOff + s * C::kTileBytes + a * 16384, w ? &tm_v : &tm_k,
                        &kv_full[s], a * 64, sp.k0 + j * 128, zkv);
          ++issued;
        }
      }
      // Let every copy this thread started land before the CTA can exit.
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (n_t(t) > 0) mbar_wait_drain(&q_full[t], 0);
      const uint32_t first = issued > (uint32_t)NS ? issued - NS : 0u;
      for (uint32_t i = first; i < issued; ++i) mbar_wait_drain(&kv_full[i % NS], (i / NS) & 1u);
    } else if (warp == 9 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);
      auto issue_qk = [&](int t, uint32_t slot) {
        const SDesc qd = sdesc_sw128_split(sbase + C::kQOff + t * C::kTileBytes, 16, 1024);
        const SDesc kd = sdesc_sw128_split(sbase + C::kKVOff + slot * C::kTileBytes, 16, 1024);
        mma_ss_w<0>(tmem + t * 128, qd.lo, qd.hi, kd.lo, kd.hi, kIdescQK);
#pragma unroll
        for (int kk = 1; kk < D / 16; ++kk) {
          const uint32_t o = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          mma_ss_w<1>(tmem + t * 128, qd.lo + o, qd.hi, kd.lo + o, kd.hi, kIdescQK);
        }
      };
      auto issue_pv = [&](int t, uint32_t slot, bool acc) {
        const SDesc vd = sdesc_sw128_split(sbase + C::kKVOff + slot * C::kTileBytes, 16384, 1024);
        const uint32_t pa = tmem + t * 128 + 64, od = tmem + 256 + t * 128;
        mma_ts_w<-1>(od, pa, vd.lo, vd.hi, kIdescPV, acc ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk) mma_ts_w<1>(od, pa + kk * 8, vd.lo + kk * 128, vd.hi, kIdescPV);
      };
      auto kv_wait = [&](uint32_t idx) {
        return mbar_wait(&kv_full[idx % NS], (idx / NS) & 1u, abort_flag, kSiteKVFull);
      };

      bool ok = true;
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (ok && n_t(t) > 0) ok = mbar_wait(&q_full[t], 0, abort_flag, kSiteQFull);
      // Ring positions: K_j at 2 (j - jb), V_j at 2 (j - jb) + 1.
      if (ok && n_span > 0) ok = kv_wait(0);
      if (ok && n_span > 0) {
        tc_fence_after();
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (n_t(t) > 0 && lo_t(t) == jb) {
            issue_qk(t, 0);
            tc_commit(&s_full[t]);
          }
        tc_commit(&kv_empty[0]);
      }
      for (int j = jb; ok && j < jb + n_span; ++j) {
        const uint32_t iv = 2 * (j - jb) + 1, ik = 2 * (j - jb) + 2;
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
        for (int t = 0; t < 2; ++t) {
          if (n_t(t) == 0) continue;
          if (j >= lo_t(t) && j <= hi_t(t)) {
            if (!mbar_wait(&p_full[t], (j - lo_t(t)) & 1, abort_flag, kSitePFull)) { ok = false; break; }
            tc_fence_after();
            issue_pv(t, iv % NS, j > lo_t(t));
            if (j == hi_t(t)) {
              tc_commit(&o_full[t]);
            } else {
              if (!need_k_next()) { ok = false; break; }
              issue_qk(t, ik % NS);
              tc_commit(&s_full[t]);
            }
          } else if (lo_t(t) == j + 1) {
            // This tile's first key tile is the next one.
            if (!need_k_next()) { ok = false; break; }
            issue_qk(t, ik % NS);
            tc_commit(&s_full[t]);
          }
        }
        // K_{j+1} feeds some tile whenever j + 1 is in the span (the two tiles'
        // ranges overlap or touch); release its slot even if no tile used it.
        if (ok && j + 1 < jb + n_span && !need_k_next()) ok = false;
        if (!ok) break;
        tc_commit(&kv_empty[iv % NS]);
        if (k_ready) tc_commit(&kv_empty[ik % NS]);
      }
      // Let this thread's MMAs finish before TMEM can be released.
      if (n_span > 0) {                       // nothing to drain when no tile was issued
        tc_commit(mma_done);
        mbar_wait_drain(mma_done, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    regs_grow<kFwdRegsSoftmax>();
    const int t = warp >> 2;
    const int quad = warp & 3;
    const int row = m0 + t * 128 + quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t t_s = tmem + lane_base + t * 128;
    const uint32_t t_p = t_s + 64;
    const uint32_t t_o = tmem + lane_base + 256 + t * 128;
    const int n = n_t(t);
    const int r_first = m0 + t * 128;                        // first and last row of this tile
    const int r_last = min(r_first + 127, Nq - 1);
    // Visible keys of this row: [k_lo, k_hi] (k_hi < k_lo: none).
    const int k_lo = (MODE == kMaskGeneral) ? max(0, win.lo(row)) : 0;
    const int k_hi = (MODE == kMaskGeneral) ? min(Nk - 1, win.hi(row))
                                            : ((MODE == kMaskCausal) ? min(row, Nk - 1) : Nk - 1);
    const bool ragged = (Nk & 127) != 0;

    float m_run = -INFINITY;   // running max, log2 units (scaled logits * log2 e)
    float l_run = 0.f;         // running sum of 2^(t - m_run), unrounded (for lse)
    float l_mma = 0.f;         // running sum of the bf16-rounded P fed to the MMA (for O)
    bool ok = n > 0;
    for (int jj = 0; ok && jj < n; ++jj) {
      const int j = lo_t(t) + jj;                            // key tile
      const int kb = j * 128;
      if (!mbar_wait(&s_full[t], jj & 1, abort_flag, kSiteSFull)) { ok = false; break; }
      tc_fence_after();
      uint32_t r0[32], r1[32], r2[32], r3[32];
      tmem_ld32(t_s + 0, r0);
      tmem_ld32(t_s + 32, r1);
      tmem_ld32(t_s + 64, r2);
      tmem_ld32(t_s + 96, r3);
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
      // All 128 scores are exponentiated into 64 packed bf16 pairs first and
      // stored with two 32-column TMEM stores at the end: a store after every
      // 32 columns made each chunk wait for its last exponential before the
      // next chunk started (measured 4 % slower on 16K-key rows). The S
      // registers die as the P words are produced, so the peak stays near 150
      // registers. Two row sums are kept. The exact one (unrounded p, paired
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
      emit(r0, 0);
      emit(r1, 16);
      emit(r2, 32);
      emit(r3, 48);
      tmem_st32(t_p, *reinterpret_cast<const uint32_t(*)[32]>(pall));
      tmem_st32(t_p + 32, *reinterpret_cast<const uint32_t(*)[32]>(pall + 32));
      const float2 ex = fadd2(ex0, ex1);
      l_run += ex.x + ex.y;
      l_mma += (q0 + q1) + (q2 + q3);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }

    // Epilogue. A row that saw no key (l = 0) gets O = 0 and lse = -inf.
    // Tile 1 of a one-tile CTA holds rows of the next CTA: never write them.
    const bool present = r_first < Nq && (t == 0 || !one_tile);
    if (ok) ok = mbar_wait(&o_full[t], 0, abort_flag, kSiteOFull);
    const bool write = ok || (present && n == 0);
    // The warpgroup writes its tile through shared memory and a TMA store when
    // every thread may write and the tile is whole (the fixed layout clips rows
    // past Nq through the tensor map). Q_t's slot is free: tile t's last S MMA
    // finished before o_full[t]. Otherwise each thread stores its own row.
    const bool all_write = named_barrier_and(1 + t, 128, write);
    const bool tma_tile = present && (!PACKED || r_first + 128 <= Nq);
    const bool has_o = n > 0;
    const float inv_l = (l_mma > 0.f) ? 1.0f / l_mma : 0.f;
    if (all_write && tma_tile) {
      if (has_o) tc_fence_after();
      uint8_t* tile = smem + C::kQOff + t * C::kTileBytes;
      const int tr = quad * 32 + lane;                       // row within the tile
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (has_o) {
          tmem_ld32(t_o + c * 32, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(u2f(o[2 * e]) * inv_l, u2f(o[2 * e + 1]) * inv_l);
        uint8_t* rowp = tile + (c >> 1) * 16384 + tr * 128;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int ch = (c & 1) * 4 + qq;
          *reinterpret_cast<uint4*>(rowp + ((ch ^ (tr & 7)) << 4)) =
              make_uint4(pk[4 * qq], pk[4 * qq + 1], pk[4 * qq + 2], pk[4 * qq + 3]);
        }
      }
      fence_proxy_async_smem();
      named_barrier_sync(1 + t, 128);
      if (quad == 0 && lane == 0) {
#pragma unroll
        for (int a = 0; a < D / 64; ++a)
          tma_store_3d(&tm_o, tile + a * 16384, a * 64, sp.q0 + r_first, zq);
        bulk_commit_group();
        bulk_wait_read_all();
      }
    } else if (write) {
      if (has_o) tc_fence_after();
      const long long o_z = PACKED ? geom.o_z : static_cast<long long>(Nq) * D;
      const long long o_row = PACKED ? geom.o_row : D;
      __nv_bfloat16* orow = out + zq * o_z + (sp.q0 + (row < Nq ? row : 0)) * o_row;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (has_o) {
          tmem_ld32(t_o + c * 32, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(u2f(o[2 * e]) * inv_l, u2f(o[2 * e + 1]) * inv_l);
        if (row < Nq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
          dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
        }
      }
    }
    if (write && row < Nq)
      lse_out[zq * (PACKED ? geom.lse_z : static_cast<long long>(Nq)) + sp.q0 + row] =
          (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
