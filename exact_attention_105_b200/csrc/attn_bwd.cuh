// Backward kernels: dQ, dK, dV of O = softmax(Q K^T * scale [causal]) V.
//
// The pages give the forward formula only (hysenlabs.com "FlashAttention:
// exakte Attention-Kernel fuer CUDA und ROCm", section "Die Schnittstellen
// von flash_attn_func bis KV-Cache"), and list fwd+bwd among the upstream
// kernels' features. The gradient computed here is the exact gradient of
// that formula:
//   P = exp(scale * Q K^T - lse)   (recomputed per tile from q, k and lse)
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  D = rowsum(dO * O)
//   dQ = scale * dS K,  dK = scale * dS^T Q
// D = rowsum(dO * O) equals rowsum(P * dP) because O = P V.
//
// Three kernels, all deterministic (no atomics):
//   bwd_pre_kernel   -D and -lse * log2(e), per query row, into the workspace
//                    (negated so P and dS are one paired fma/add each),
//                    padded to a multiple of 128 rows per head. Padding rows
//                    get -lse = -inf, so every P that involves them is 0.
//   bwd_dkdv_kernel  one CTA per (batch, KV head, 128-key block). K_j and V_j
//                    stay in shared memory. It loops over the 128-query blocks
//                    of every query head in the GQA group (from the diagonal
//                    when causal). Per block it computes S^T, dP^T, P^T, dS^T
//                    and accumulates dV and dK in TMEM: S^T (then P^T) in
//                    columns [0, 128), dP^T (then dS^T) in [128, 256), dV in
//                    [256, 256 + d), dK in [384, 512). At d = 64 the free
//                    columns hold a second S^T buffer ([384, 512), dK moves to
//                    [320, 384)) for odd steps, so S^T(s+2) is issued right
//                    after dV(s) and the compute warps find S^T(s+1) ready.
//   bwd_dq_kernel    one CTA per (batch, query head, 128-query block). Q_i and
//                    dO_i stay resident while K_j and V_j stream through two
//                    rings (K_j is held from S(j) to dQ(j), V_j only for dP(j)).
//                    Per key block it computes S, dP, P, dS and accumulates dQ
//                    in TMEM: S in columns [0, 128), dQ in [256, 384), and dP
//                    of block j, overwritten by its dS, in [128, 256) for even
//                    j and [384, 512) for odd j. With two dP buffers, dP(j+1)
//                    is issued right after S(j+1), ahead of dQ(j), and waits
//                    only for dQ(j-1), which read the same buffer.
// Warp roles in both main kernels (384 threads): warps 0-7 are two compute
// warpgroups, warp 8 is the TMA producer, warp 9 allocates TMEM and issues
// the MMAs, and warps 10-11 idle. Thread r of a compute warpgroup owns TMEM
// lane r. Warpgroup h owns columns [64h, 64h+64) of the step's 128x128 S and
// dP tiles. It writes its bf16 P/dS pairs back into the first 32 of its own
// 64 columns, so neither group overwrites columns the other has yet to read.
// The MMA that consumes them reads K-step kk (16 columns) from TMEM column
// 64*(kk/4) + 8*(kk%4) of the tile.
// Both kernels end by staging their bf16 output tile (dK and dV, or dQ) in
// shared memory that no MMA reads any more (the K/V tiles, or the Q tile),
// 128-byte swizzled, and writing it with TMA stores. Packed tiles that run
// past their sequence are written row by row instead, since the tensor map
// only bounds the whole packed tensor.
#pragma once

#include "geometry.cuh"
#include "sm100.cuh"
#include "visibility.cuh"

namespace attn {

constexpr float kLog2e = 1.4426950408889634f;
// Work counters at the end of the workspace: [0] dK/dV items, [1] dQ items.
constexpr int kBwdCounters = 2;
constexpr size_t kBwdCounterBytes = 64;

__host__ __device__ inline int pad128(int n) { return (n + 127) & ~127; }

// ------------------------------------------------------------------ preprocess
// 8 lanes per query row, 4 rows per warp, 32 rows per 256-thread block. The
// grid covers B * Hq * Npad workspace rows exactly (Npad a multiple of 128),
// so every shuffle group is fully populated. Workspace row (b * Hq + h) * Npad
// + n holds query n of sequence b, head h; rows past the sequence get
// -lse*log2(e) = -inf (so P = 0 there) and D = 0. It also zeroes the two
// work counters of the persistent kernels that follow it on the stream.
template <int D>
__global__ void __launch_bounds__(256)
bwd_pre_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
               const float* __restrict__ lse, float* __restrict__ L, float* __restrict__ Dv,
               int Hq, SeqGeom geom, int Npad, int* __restrict__ sched) {
  grid_dep_wait();     // o and lse may come from the kernel just before
  if (blockIdx.x == 0 && threadIdx.x < kBwdCounters) sched[threadIdx.x] = 0;
  const long long row = static_cast<long long>(blockIdx.x) * 32 + (threadIdx.x >> 3);
  const int sub = threadIdx.x & 7;
  const long long bh = row / Npad;
  const int n = static_cast<int>(row - bh * Npad);
  const int b = static_cast<int>(bh / Hq);
  const int h = static_cast<int>(bh - static_cast<long long>(b) * Hq);
  const SeqSpan sp = geom.cu_q ? seq_span<true>(geom, b) : seq_span<false>(geom, b);
  const long long z = geom.cu_q ? h : bh;
  const int N = sp.nq;
  float acc = 0.f;
  if (n < N) {
    constexpr int kPer = D / 8;  // elements per lane: 16 (D=128) or 8 (D=64)
    const size_t base = z * geom.o_z + (sp.q0 + n) * geom.o_row + sub * kPer;
    const uint4* po = reinterpret_cast<const uint4*>(o + base);
    const uint4* pd = reinterpret_cast<const uint4*>(dO + base);
#pragma unroll
    for (int v = 0; v < kPer / 8; ++v) {
      const uint4 a = po[v], b = pd[v];
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(u2f(aw[e] << 16), u2f(bw[e] << 16), acc);
        acc = fmaf(u2f(aw[e] & 0xFFFF0000u), u2f(bw[e] & 0xFFFF0000u), acc);
      }
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  if (sub == 0) {
    const float l = (n < N) ? lse[z * geom.lse_z + sp.q0 + n] : -INFINITY;
    // A row that saw no key (lse = -inf) is treated like padding: P = 0.
    L[row] = (l == -INFINITY) ? -INFINITY : -l * kLog2e;
    Dv[row] = (n < N) ? -acc : 0.f;
  }
  grid_dep_launch();
}

// ------------------------------------------------------------------ shared bits
enum BwdSite : int {
  kSiteBKV = 0x11, kSiteBLoadFull = 0x12, kSiteBLoadEmpty = 0x13, kSiteBS = 0x14,
  kSiteBDP = 0x15, kSiteBP = 0x16, kSiteBDS = 0x17, kSiteBAcc = 0x18, kSiteBSFree = 0x19,
  kSiteBItem = 0x1A, kSiteBStage = 0x1B
};

// Loads a 128-column fp32 row block from TMEM into four 32-register blocks.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r0)[32], uint32_t (&r1)[32],
                                           uint32_t (&r2)[32], uint32_t (&r3)[32]) {
  tmem_ld32(taddr + 0, r0);
  tmem_ld32(taddr + 32, r1);
  tmem_ld32(taddr + 64, r2);
  tmem_ld32(taddr + 96, r3);
  tmem_ld_wait(r0);
  reg_fence(r1);
  reg_fence(r2);
  reg_fence(r3);
}

// dS = P * (dP - D) for 32 columns, P in fp32, given -D per column pair as
// float2 through `nd(e)` (e even); writes 16 packed bf16 pairs of dS.
template <typename NegD>
__device__ __forceinline__ void ds_block(const float* pf, const uint32_t (&dp)[32],
                                         uint32_t* out, NegD nd) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float2 d = fadd2(make_float2(u2f(dp[2 * e]), u2f(dp[2 * e + 1])), nd(2 * e));
    const float2 v = fmul2(make_float2(pf[2 * e], pf[2 * e + 1]), d);
    out[e] = pack_bf16x2(v.x, v.y);
  }
}

// TMEM column offset of K-step kk (16 bf16 columns) of a P / dS tile whose
// two 64-column halves were packed into the first 32 columns of each half.
__device__ __forceinline__ uint32_t split_col(int kk) { return 64 * (kk >> 2) + 8 * (kk & 3); }

// Epilogue helper: one 128 x D fp32 accumulator row (this thread's lane) ->
// bf16 * mul, stored to `dst` when `valid`.
template <int D, int C0 = 0, int C1 = D / 32>
__device__ __forceinline__ void store_acc_row(uint32_t t_acc, __nv_bfloat16* dst, float mul,
                                              bool valid) {
#pragma unroll
  for (int c = C0; c < C1; ++c) {
    uint32_t a[32];
    tmem_ld32(t_acc + c * 32, a);
    tmem_ld_wait(a);
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(u2f(a[2 * e]) * mul, u2f(a[2 * e + 1]) * mul);
    if (valid) {
      uint4* p = reinterpret_cast<uint4*>(dst + c * 32);
      p[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      p[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      p[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
      p[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
    }
  }
}

// Epilogue helper: this thread's 128 x D fp32 accumulator row (tile row t)
// -> bf16 * mul into a shared-memory tile laid out as the 128-byte-swizzled
// TMA box expects: D/64 blocks of 128 rows x 128 bytes, the 16-byte chunk c
// of row t at chunk position c ^ (t & 7).
template <int D, int C0 = 0, int C1 = D / 32>
__device__ __forceinline__ void stage_acc_row(uint32_t t_acc, uint8_t* tile, int t, float mul) {
#pragma unroll
  for (int cc = C0; cc < C1; ++cc) {
    uint32_t a[32];
    tmem_ld32(t_acc + cc * 32, a);
    tmem_ld_wait(a);
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(u2f(a[2 * e]) * mul, u2f(a[2 * e + 1]) * mul);
    uint8_t* rowp = tile + (cc >> 1) * 16384 + t * 128;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = (cc & 1) * 4 + q;
      *reinterpret_cast<uint4*>(rowp + ((c ^ (t & 7)) << 4)) =
          make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    }
  }
}

// ------------------------------------------------------------------ dK / dV
// Persistent. The work items are (batch, KV head, 128-key block), numbered
// head-major with the key block fastest: CTAs running at the same time mostly
// share one head's Q and dO in L2, and within a head the causal key blocks
// with the most query blocks come first. The last `tail_heads` heads are
// numbered key-block-major instead, so the last items handed out are the
// lightest ones of several heads and the CTAs finish close together. Each
// CTA starts with item blockIdx.x and then takes gridDim.x + the next value
// of a counter in the workspace (zeroed by bwd_pre_kernel), so CTAs that
// finish early take more items. The producer passes every item to the other roles through a
// two-slot ring in shared memory; a value of -1 ends the kernel.
// An item's K and V are released as soon as its last S^T and dP^T MMAs have
// run, so the next item's K and V load during its last step. Its dK and dV
// are staged in the shared memory of its last (Q, dO) stage (by then read by
// no MMA) and written by the store warp, which then releases that stage. The
// next item's first MMAs run meanwhile: they touch neither that stage nor the
// accumulator columns that the epilogue reads, and its first dV MMA (which
// overwrites the accumulator) waits for P, which the compute warps produce
// only after their epilogue has read dK and dV.
template <int D>
struct DkdvCfg {
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kStages = (D == 128) ? 2 : 4;     // (Q_i, dO_i, L_i, D_i) stages
  static constexpr int kItemSlots = 2;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTile;
  static constexpr int kStageOff = 2 * kTile;
  static constexpr int kStageBytes = 2 * kTile + 1024;   // Q, dO, 128 L floats, 128 D floats
  static constexpr int kBarOff = kStageOff + kStages * kStageBytes;
  // kv_full kv_empty ld_full[S] ld_empty[S] s_full dp_full p_full ds_full acc_full
  // stage_full item_full[I] item_empty[I] mma_done s_full2
  static constexpr int kNumBars = 2 + 2 * kStages + 6 + 2 * kItemSlots + 1 + 1;
  // d = 64 leaves 128 tensor-memory columns free: S^T is double-buffered
  // there (columns [384, 512)), with dK moved to [320, 384).
  static constexpr bool kDB = D == 64;
  static constexpr int kDkCol = kDB ? 320 : 384;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 8 + 4 * kItemSlots;  // TMEM slot, abort flag, items
  static constexpr int kSmemAlloc = kBytes + 1024;
  static constexpr int kThreads = 384;
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
};

// Readers of each item slot: the MMA thread, the 8 compute warps (one lane
// each) and the store thread.
constexpr int kItemReaders = 10;

struct DkdvItem {
  SeqSpan sp;
  int b, hkv, j, zkv, i_start, per_head;
  int n_steps;  // query blocks to visit (0: no query sees these keys; -1: past the keys)
};

template <int MODE, bool PACKED>
__device__ __forceinline__ DkdvItem dkdv_item(int item, int Hkv, int group, int nkv,
                                              int tail_heads, int n_items, const SeqGeom& geom,
                                              KeyWindow win) {
  DkdvItem it;
  const int split = n_items - tail_heads * nkv;
  int bh_kv;
  if (item < split) {
    bh_kv = item / nkv;
    it.j = item - bh_kv * nkv;
  } else {
    const int r = item - split;
    it.j = r / tail_heads;
    bh_kv = split / nkv + (r - it.j * tail_heads);
  }
  it.b = bh_kv / Hkv;
  it.hkv = bh_kv - it.b * Hkv;
  it.zkv = PACKED ? it.hkv : bh_kv;
  it.sp = seq_span<PACKED>(geom, it.b);
  win.off = it.sp.nk - it.sp.nq;              // bottom-right alignment per sequence
  int i_end;
  q_block_range<MODE>(it.j, it.sp.nq, it.sp.nk, win, it.i_start, i_end);
  it.per_head = max(0, i_end - it.i_start + 1);
  it.n_steps = (it.j * 128 < it.sp.nk) ? group * it.per_head : -1;
  return it;
}

template <int D, int MODE, int FEAT>
__global__ void __launch_bounds__(384, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_dk,
                const __grid_constant__ CUtensorMap tm_dv,
                const float* __restrict__ Lws, const float* __restrict__ Dws,
                __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv, int Hq, int group,
                SeqGeom geom, int Npad, float scale_log2, float scale, KeyWindow win,
                Softcap cap, int* __restrict__ sched, int n_items, int tail_heads) {
  constexpr bool SOFTCAP = (FEAT & kFeatSoftcap) != 0;
  constexpr bool PACKED = (FEAT & kFeatPacked) != 0;
  static_assert(FEAT == 0 || MODE == kMaskGeneral, "features run in the general mode");
  using C = DkdvCfg<D>;
  constexpr int NS = C::kStages;
  constexpr int IS = C::kItemSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + 1;       // the item's last S^T and dP^T MMAs are done
  uint64_t* ld_full = kv_empty + 1;
  uint64_t* ld_empty = ld_full + NS;
  uint64_t* s_full = ld_empty + NS;
  uint64_t* dp_full = s_full + 1;
  uint64_t* p_full = dp_full + 1;
  uint64_t* ds_full = p_full + 1;
  uint64_t* acc_full = ds_full + 1;       // the item's dK and dV are complete in TMEM
  uint64_t* stage_full = acc_full + 1;    // the item's dK and dV are staged (or stored)
  uint64_t* item_full = stage_full + 1;
  uint64_t* item_empty = item_full + IS;
  uint64_t* mma_done = item_empty + IS;
  uint64_t* s_full2 = mma_done + 1;       // double-buffered mode: S^T of odd steps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 8);
  constexpr bool DB = C::kDB;
  // S^T buffer and its barrier for step g.
  auto s_col = [&](uint32_t g) { return (DB && (g & 1)) ? 384u : 0u; };
  auto s_bar = [&](uint32_t g) { return (DB && (g & 1)) ? s_full2 : s_full; };
  auto s_par = [&](uint32_t g) { return DB ? (g >> 1) & 1u : g & 1u; };

  const int warp = warp_id(), lane = lane_id();
  const int Hkv = Hq / group;
  const int nkv = (geom.Nk + 127) >> 7;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&ld_full[s], 1);
      mbar_init(&ld_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 256);
    mbar_init(ds_full, 256);
    mbar_init(acc_full, 1);
    mbar_init(stage_full, 1);
    for (int s = 0; s < IS; ++s) {
      mbar_init(&item_full[s], 1);
      mbar_init(&item_empty[s], kItemReaders);
    }
    mbar_init(mma_done, 1);
    mbar_init(s_full2, 1);
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

  // Item k of this CTA, as published by the producer (-1: no more).
  auto read_item = [&](int k, int& item) {
    if (!mbar_wait(&item_full[k % IS], (k / IS) & 1, abort_flag, kSiteBItem)) return false;
    item = item_slot[k % IS];
    return true;
  };
  auto step_head = [&](const DkdvItem& it, int s, int& i, int& bh_q) {
    const int g = s / it.per_head;
    i = it.i_start + (s - g * it.per_head);
    bh_q = it.b * Hq + it.hkv * group + g;
  };

  if (warp == 8) {
    if (lane == 0) {
      // -------------------------------------------------------- producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      uint32_t g = 0;            // (Q, dO) loads issued: the ring position of the next
      int kv_loads = 0;          // items whose K and V were loaded
      int item = blockIdx.x;
      int next = -1;             // the following item, fetched one item ahead
      bool ok = true;
      for (int k = 0; ok; ++k) {
        DkdvItem it;
        while (item < n_items) {   // skip numbers past a packed sequence's keys
          it = dkdv_item<MODE, PACKED>(item, Hkv, group, nkv, tail_heads, n_items, geom, win);
          if (it.n_steps >= 0) break;
          item = next >= 0 ? next : gridDim.x + atomicAdd(sched, 1);
          next = -1;
        }
        const bool done = item >= n_items;
        const int slot = k % IS;
        if (k >= IS && !mbar_wait(&item_empty[slot], ((k / IS) - 1) & 1, abort_flag, kSiteBItem)) {
          ok = false;
          break;
        }
        item_slot[slot] = done ? -1 : item;
        mbar_arrive(&item_full[slot]);
        if (done) break;
        if (next < 0) next = gridDim.x + atomicAdd(sched, 1);
        if (it.n_steps > 0) {
          if (kv_loads > 0 && !mbar_wait(kv_empty, (kv_loads - 1) & 1, abort_flag, kSiteBKV)) {
            ok = false;
            break;
          }
          mbar_expect_tx(kv_full, 2 * C::kTile);
#pragma unroll
          for (int a = 0; a < D / 64; ++a) {
            tma_load_3d(smem + C::kKOff + a * 16384, &tm_k, kv_full, a * 64,
                        it.sp.k0 + it.j * 128, it.zkv);
            tma_load_3d(smem + C::kVOff + a * 16384, &tm_v, kv_full, a * 64,
                        it.sp.k0 + it.j * 128, it.zkv);
          }
          ++kv_loads;
          for (int s = 0; s < it.n_steps; ++s, ++g) {
            const int st = g % NS;
            const uint32_t round = g / NS;
            if (round > 0 &&
                !mbar_wait(&ld_empty[st], (round - 1) & 1u, abort_flag, kSiteBLoadEmpty)) {
              ok = false;
              break;
            }
            int i, bh_q;
            step_head(it, s, i, bh_q);
            const int zq = PACKED ? bh_q - it.b * Hq : bh_q;
            uint8_t* stage = smem + C::kStageOff + st * C::kStageBytes;
            mbar_expect_tx(&ld_full[st], 2 * C::kTile + 1024);
#pragma unroll
            for (int a = 0; a < D / 64; ++a) {
              tma_load_3d(stage + a * 16384, &tm_q, &ld_full[st], a * 64, it.sp.q0 + i * 128, zq);
              tma_load_3d(stage + C::kTile + a * 16384, &tm_do, &ld_full[st], a * 64,
                          it.sp.q0 + i * 128, zq);
            }
            const size_t off = static_cast<size_t>(bh_q) * Npad + i * 128;
            bulk_load(stage + 2 * C::kTile, Lws + off, 512, &ld_full[st]);
            bulk_load(stage + 2 * C::kTile + 512, Dws + off, 512, &ld_full[st]);
          }
        }
        item = next;
        next = -1;
      }
      // Let every copy this thread started land before the CTA can exit.
      if (kv_loads > 0) mbar_wait_drain(kv_full, (kv_loads - 1) & 1);
      for (uint32_t x = g > static_cast<uint32_t>(NS) ? g - NS : 0u; x < g; ++x)
        mbar_wait_drain(&ld_full[x % NS], (x / NS) & 1u);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // -------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, 0, 1);
      auto stage_addr = [&](uint32_t g) { return sbase + C::kStageOff + (g % NS) * C::kStageBytes; };
      // dst(tmem) = A_kmajor(smem tile) * B_kmajor(smem tile)^T, K = D
      auto mma_tile_kk = [&](uint32_t dst, uint32_t a, uint32_t bt) {
        const SDesc ad = sdesc_sw128_split(a, 16, 1024), bd = sdesc_sw128_split(bt, 16, 1024);
        mma_ss_w<0>(dst, ad.lo, ad.hi, bd.lo, bd.hi, kIdescSS);
#pragma unroll
        for (int kk = 1; kk < D / 16; ++kk) {
          const uint32_t o = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          mma_ss_w<1>(dst, ad.lo + o, ad.hi, bd.lo + o, bd.hi, kIdescSS);
        }
      };
      // acc(tmem) += A(tmem, 128 x 128 bf16, split layout) * B(smem tile, MN-major), K = 128
      auto mma_acc = [&](uint32_t acc, uint32_t a_tmem, uint32_t b, bool accumulate) {
        const SDesc bd = sdesc_sw128_split(b, 16384, 1024);
        mma_ts_w<-1>(acc, a_tmem + split_col(0), bd.lo, bd.hi, kIdescAcc, accumulate ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk)
          mma_ts_w<1>(acc, a_tmem + split_col(kk), bd.lo + kk * 128, bd.hi, kIdescAcc);
      };
      uint32_t g = 0;            // steps issued over all items (ring position)
      int kv_loads = 0;
      bool ok = true, any = false;
      for (int k = 0; ok; ++k) {
        int item;
        if (!read_item(k, item)) { ok = false; break; }
        mbar_arrive(&item_empty[k % IS]);
        if (item < 0) break;
        const DkdvItem it = dkdv_item<MODE, PACKED>(item, Hkv, group, nkv, tail_heads, n_items, geom, win);
        const int n = it.n_steps;
        if (n <= 0) continue;
        if (!mbar_wait(kv_full, kv_loads & 1, abort_flag, kSiteBKV) ||
            !mbar_wait(&ld_full[g % NS], (g / NS) & 1u, abort_flag, kSiteBLoadFull)) {
          ok = false;
          break;
        }
        ++kv_loads;
        any = true;
        tc_fence_after();
        mma_tile_kk(tmem + s_col(g), sbase + C::kKOff, stage_addr(g));          // S^T(0)
        tc_commit(s_bar(g));
        mma_tile_kk(tmem + 128, sbase + C::kVOff, stage_addr(g) + C::kTile);    // dP^T(0)
        tc_commit(dp_full);
        if (DB && n > 1) {
          // S^T(1) into the second buffer right away.
          if (!mbar_wait(&ld_full[(g + 1) % NS], ((g + 1) / NS) & 1u, abort_flag,
                         kSiteBLoadFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_tile_kk(tmem + s_col(g + 1), sbase + C::kKOff, stage_addr(g + 1));
          tc_commit(s_bar(g + 1));
        }
        if (n == 1) tc_commit(kv_empty);
        for (int s = 0; ok && s < n; ++s, ++g) {
          const uint32_t sa = stage_addr(g);
          if (!mbar_wait(p_full, g & 1u, abort_flag, kSiteBP)) { ok = false; break; }
          tc_fence_after();
          mma_acc(tmem + 256, tmem + s_col(g), sa + C::kTile, s > 0);             // dV += P^T dO
          const bool more = s + 1 < n;
          // S^T of a later step: the next one (single buffer, after dV has
          // read P^T from its columns), or the one after (double-buffered).
          const uint32_t gn = DB ? g + 2 : g + 1;
          if (DB ? s + 2 < n : more) {
            if (!mbar_wait(&ld_full[gn % NS], (gn / NS) & 1u, abort_flag, kSiteBLoadFull)) {
              ok = false;
              break;
            }
            tc_fence_after();
            mma_tile_kk(tmem + s_col(gn), sbase + C::kKOff, stage_addr(gn));     // S^T
            tc_commit(s_bar(gn));
          }
          if (!mbar_wait(ds_full, g & 1u, abort_flag, kSiteBDS)) { ok = false; break; }
          tc_fence_after();
          mma_acc(tmem + C::kDkCol, tmem + 128, sa, s > 0);                       // dK += dS^T Q
          if (more) {
            // The last step's stage is released by the store thread instead.
            tc_commit(&ld_empty[g % NS]);
            mma_tile_kk(tmem + 128, sbase + C::kVOff, stage_addr(g + 1) + C::kTile); // dP^T(s+1)
            tc_commit(dp_full);
            if (s + 2 == n) tc_commit(kv_empty);
          }
        }
        if (ok) tc_commit(acc_full);
      }
      if (any) {                             // nothing to drain when nothing was issued
        tc_commit(mma_done);
        mbar_wait_drain(mma_done, 0);
      }
    }
    __syncwarp();
  } else if (warp == 10) {
    if (lane == 0) {
      // -------------------------------------------------------- output store
      tma_prefetch_desc(&tm_dk);
      tma_prefetch_desc(&tm_dv);
      uint32_t g = 0;
      int staged = 0;
      for (int k = 0;; ++k) {
        int item;
        if (!read_item(k, item)) break;
        mbar_arrive(&item_empty[k % IS]);
        if (item < 0) break;
        const DkdvItem it = dkdv_item<MODE, PACKED>(item, Hkv, group, nkv, tail_heads, n_items, geom, win);
        if (it.n_steps <= 0) continue;
        g += it.n_steps;
        if (!mbar_wait(stage_full, staged & 1, abort_flag, kSiteBStage)) break;
        ++staged;
        const int st = (g - 1) % NS;
        if (!PACKED || it.j * 128 + 128 <= it.sp.nk) {
          uint8_t* stage = smem + C::kStageOff + st * C::kStageBytes;
#pragma unroll
          for (int a = 0; a < D / 64; ++a) {
            tma_store_3d(&tm_dv, stage + C::kTile + a * 16384, a * 64, it.sp.k0 + it.j * 128,
                         it.zkv);
            tma_store_3d(&tm_dk, stage + a * 16384, a * 64, it.sp.k0 + it.j * 128, it.zkv);
          }
          bulk_commit_group();
          bulk_wait_read_all();
        }
        mbar_arrive(&ld_empty[st]);
      }
      bulk_wait_read_all();
    }
    __syncwarp();
  } else if (warp < 8) {
    // ---------------------------------------------------------- compute
    const int h = warp >> 2;                          // column half of the step tile
    const int quad = warp & 3;
    const int t = quad * 32 + lane;                   // key row within the block
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t t_s = tmem + lane_base + 64 * h;          // S^T half; P^T into +0..32
    const uint32_t t_dp = tmem + lane_base + 128 + 64 * h;   // dP^T half; dS^T into +0..32
    const int c_base = 64 * h;
    uint32_t g = 0;
    int acc_items = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int item = -1;
      if (!read_item(k, item)) ok = false;
      __syncwarp();
      if (lane == 0) mbar_arrive(&item_empty[k % IS]);
      // All compute threads agree before going on, so that every named
      // barrier below is reached by all of them or by none.
      ok = named_barrier_and(1, 256, ok);
      if (!ok || item < 0) break;
      const DkdvItem it = dkdv_item<MODE, PACKED>(item, Hkv, group, nkv, tail_heads, n_items, geom, win);
      const int j = it.j, n_steps = it.n_steps, Nq = it.sp.nq, Nk = it.sp.nk;
      const int key = j * 128 + t;
      KeyWindow w = win;
      w.off = Nk - Nq;
      // Query q sees this key iff key - off - wr <= q <= key - off + wl.
      const int q_first = key - w.off - w.wr, q_last = key - w.off + w.wl;
      for (int s = 0; ok && s < n_steps; ++s, ++g) {
        int i, bh_q;
        step_head(it, s, i, bh_q);
        const int st = g % NS;
        const float* Ls = reinterpret_cast<const float*>(smem + C::kStageOff + st * C::kStageBytes +
                                                         2 * C::kTile) + c_base;
        const float* Ds = Ls + 128;
        if (!mbar_wait(&ld_full[st], (g / NS) & 1u, abort_flag, kSiteBLoadFull) ||
            !mbar_wait(s_bar(g), s_par(g), abort_flag, kSiteBS)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t_sg = t_s + s_col(g);
        uint32_t r0[32], r1[32];
        tmem_ld32(t_sg, r0);
        tmem_ld32(t_sg + 32, r1);
        tmem_ld_wait(r0);
        reg_fence(r1);
        // Masked steps: the causal diagonal, or (general mode) query blocks at
        // an edge of the key tile's visibility band.
        bool edge;
        if (MODE == kMaskNone) edge = false;
        else if (MODE == kMaskCausal) edge = i == j;
        else edge = j * 128 < w.lo(min(i * 128 + 127, Nq - 1)) || j * 128 + 127 > w.hi(i * 128);
        const int c_lo = q_first - i * 128, c_hi = q_last - i * 128;   // keep columns [c_lo, c_hi]
        const float2 sc2 = make_float2(scale_log2, scale_log2);
        float pf[64];                                   // P in fp32 (for dS)
        uint32_t pw[32];                                // P as bf16 pairs (for the dV MMA)
        auto p_block = [&](const uint32_t (&r)[32], int c0) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = c_base + c0 + 2 * e;
            const float2 nl = *reinterpret_cast<const float2*>(&Ls[c0 + 2 * e]);
            float p0, p1, g0 = 1.f, g1 = 1.f;
            if constexpr (SOFTCAP) {
              // P from the capped logit; dS gets the chain-rule factor 1 - t^2.
              const float t0 = softcap_tanh(u2f(r[2 * e]), cap);
              const float t1 = softcap_tanh(u2f(r[2 * e + 1]), cap);
              p0 = fast_exp2(fmaf(cap.out, t0, nl.x));
              p1 = fast_exp2(fmaf(cap.out, t1, nl.y));
              g0 = fmaf(-t0, t0, 1.f);
              g1 = fmaf(-t1, t1, 1.f);
            } else {
              const float2 x = ffma2(make_float2(u2f(r[2 * e]), u2f(r[2 * e + 1])), sc2, nl);
              p0 = fast_exp2(x.x);
              p1 = fast_exp2(x.y);
            }
            if (edge) {
              if (MODE == kMaskGeneral) {
                if (c < c_lo || c > c_hi) p0 = 0.f;
                if (c + 1 < c_lo || c + 1 > c_hi) p1 = 0.f;
              } else {                                  // causal diagonal: one-sided
                if (c < c_lo) p0 = 0.f;
                if (c + 1 < c_lo) p1 = 0.f;
              }
            }
            pf[c0 + 2 * e] = SOFTCAP ? p0 * g0 : p0;
            pf[c0 + 2 * e + 1] = SOFTCAP ? p1 * g1 : p1;
            pw[c0 / 2 + e] = pack_bf16x2(p0, p1);
          }
        };
        p_block(r0, 0);
        p_block(r1, 32);
        tmem_st32(t_sg, pw);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);

        if (!mbar_wait(dp_full, g & 1u, abort_flag, kSiteBDP)) { ok = false; break; }
        tc_fence_after();
        uint32_t d0[32], d1[32];
        tmem_ld32(t_dp, d0);
        tmem_ld32(t_dp + 32, d1);
        tmem_ld_wait(d0);
        reg_fence(d1);
        uint32_t ds[32];
        ds_block(&pf[0], d0, ds,
                 [&](int e) { return *reinterpret_cast<const float2*>(&Ds[e]); });
        ds_block(&pf[32], d1, ds + 16,
                 [&](int e) { return *reinterpret_cast<const float2*>(&Ds[32 + e]); });
        tmem_st32(t_dp, ds);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(ds_full);
      }
      if (ok && n_steps > 0) ok = mbar_wait(acc_full, acc_items & 1, abort_flag, kSiteBAcc);
      // Every compute thread gets here once per item; the epilogue runs only
      // if all of them completed their waits, so the barriers below are
      // reached by all or none.
      ok = named_barrier_and(1, 256, ok);
      if (!ok) break;
      if (n_steps > 0) {
        ++acc_items;
        tc_fence_after();
        // A full tile (always in the fixed layout, where rows past N are
        // clipped by the tensor map) is staged for the store thread: dV over
        // the last stage's dO, dK over its Q. A packed tile that runs past
        // its sequence is written row by row.
        if (!PACKED || j * 128 + 128 <= Nk) {
          uint8_t* stage = smem + C::kStageOff + ((g - 1) % NS) * C::kStageBytes;
          stage_acc_row<D>(tmem + lane_base + (h == 0 ? 256 : C::kDkCol), stage + (h == 0 ? C::kTile : 0),
                           t, h == 0 ? 1.0f : scale);
          fence_proxy_async_smem();
        } else {
          const bool valid = key < Nk;
          const long long kv_z = PACKED ? geom.kv_z : static_cast<long long>(Nk) * D;
          const long long kv_row = PACKED ? geom.kv_row : D;
          const size_t row_off = it.zkv * kv_z + (it.sp.k0 + (valid ? key : 0)) * kv_row;
          if (h == 0)
            store_acc_row<D>(tmem + lane_base + 256, dv + row_off, 1.0f, valid);
          else
            store_acc_row<D>(tmem + lane_base + C::kDkCol, dk + row_off, scale, valid);
        }
        tc_fence_before();
        named_barrier_sync(1, 256);
        if (threadIdx.x == 0) mbar_arrive(stage_full);
      } else if (key < Nk) {
        // No query sees these keys: their gradients are zero.
        const long long kv_z = PACKED ? geom.kv_z : static_cast<long long>(Nk) * D;
        const long long kv_row = PACKED ? geom.kv_row : D;
        uint4* dst = reinterpret_cast<uint4*>((h == 0 ? dv : dk) + it.zkv * kv_z +
                                              (it.sp.k0 + key) * kv_row);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
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

// ------------------------------------------------------------------ dQ
// Persistent, scheduled like the dK/dV kernel. The work items are (batch,
// query head, 128-query block), numbered head-major with the heaviest causal
// block first within a head, and the last `tail_heads` heads numbered
// block-major (heaviest first) so the lightest items come last. An item's Q
// and dO are released as soon as its last S and dP MMAs have run, so the next
// item's load during its last step; its dQ is staged in the K ring slot of
// its last key block (read by no MMA once dQ is complete) and written by the
// store warp, which then releases that slot.
template <int D>
struct DqCfg {
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kKStages = 3;                     // K ring: K_j lives from S(j) to dQ(j)
  static constexpr int kVStages = (D == 128) ? 2 : 3;    // V ring: V_j lives for dP(j) only
  static constexpr int kItemSlots = 2;
  static constexpr int kQOff = 0;
  static constexpr int kDOOff = kTile;
  static constexpr int kKOff = 2 * kTile;
  static constexpr int kVOff = kKOff + kKStages * kTile;
  static constexpr int kBarOff = kVOff + kVStages * kTile;
  // qd_full qd_empty k_full[KS] k_empty[KS] v_full[VS] v_empty[VS] s_full s_free
  // dp_full[2] ds_full[2] acc_full stage_full item_full[I] item_empty[I] mma_done
  static constexpr int kNumBars = 2 + 2 * kKStages + 2 * kVStages + 8 + 2 * kItemSlots + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 8 + 4 * kItemSlots;  // TMEM slot, abort flag, items
  static constexpr int kSmemAlloc = kBytes + 1024;
  static constexpr int kThreads = 384;
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
};

struct DqItem {
  SeqSpan sp;
  int b, hq, bh, i, zq, zkv, j_lo;
  int n;  // key blocks to visit (0: the rows see no key; -1: past the sequence's rows)
};

template <int MODE, bool PACKED>
__device__ __forceinline__ DqItem dq_item(int item, int Hq, int group, int nqb, int tail_heads,
                                          int n_items, const SeqGeom& geom, KeyWindow win) {
  DqItem it;
  const int split = n_items - tail_heads * nqb;
  int r;  // rank of the block within its head, heaviest first
  if (item < split) {
    it.bh = item / nqb;
    r = item - it.bh * nqb;
  } else {
    const int x = item - split;
    r = x / tail_heads;
    it.bh = split / nqb + (x - r * tail_heads);
  }
  it.i = nqb - 1 - r;
  it.b = it.bh / Hq;
  it.hq = it.bh - it.b * Hq;
  it.sp = seq_span<PACKED>(geom, it.b);
  it.zq = PACKED ? it.hq : it.bh;
  it.zkv = PACKED ? it.hq / group : it.b * (Hq / group) + it.hq / group;
  win.off = it.sp.nk - it.sp.nq;             // bottom-right alignment per sequence
  int j_hi;
  kv_tile_range<MODE>(it.i * 128, min(it.i * 128 + 127, it.sp.nq - 1), it.sp.nk, win, it.j_lo,
                      j_hi);
  it.n = (it.i * 128 < it.sp.nq) ? max(0, j_hi - it.j_lo + 1) : -1;
  return it;
}

template <int D, int MODE, int FEAT>
__global__ void __launch_bounds__(384, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_dq,
              const float* __restrict__ Lws, const float* __restrict__ Dws,
              __nv_bfloat16* __restrict__ dq, int Hq, int group, SeqGeom geom, int Npad,
              float scale_log2, float scale, KeyWindow win, Softcap cap,
              int* __restrict__ sched, int n_items, int tail_heads) {
  constexpr bool SOFTCAP = (FEAT & kFeatSoftcap) != 0;
  constexpr bool PACKED = (FEAT & kFeatPacked) != 0;
  static_assert(FEAT == 0 || MODE == kMaskGeneral, "features run in the general mode");
  using C = DqCfg<D>;
  constexpr int KS = C::kKStages, VS = C::kVStages, IS = C::kItemSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* qd_full = bars;
  uint64_t* qd_empty = qd_full + 1;          // the item's last S and dP MMAs are done
  uint64_t* k_full = qd_empty + 1;
  uint64_t* k_empty = k_full + KS;
  uint64_t* v_full = k_empty + KS;
  uint64_t* v_empty = v_full + VS;
  uint64_t* s_full = v_empty + VS;
  uint64_t* s_free = s_full + 1;
  uint64_t* dp_full = s_free + 1;            // [2]: dP buffer b holds a new step
  uint64_t* ds_full = dp_full + 2;           // [2]: dS written into buffer b
  uint64_t* acc_full = ds_full + 2;          // the item's dQ is complete in TMEM
  uint64_t* stage_full = acc_full + 1;       // the item's dQ is staged (or stored)
  uint64_t* item_full = stage_full + 1;
  uint64_t* item_empty = item_full + IS;
  uint64_t* mma_done = item_empty + IS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 8);

  const int warp = warp_id(), lane = lane_id();
  const int nqb = (geom.Nq + 127) >> 7;

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    mbar_init(qd_empty, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 256);
    for (int b2 = 0; b2 < 2; ++b2) {
      mbar_init(&dp_full[b2], 1);
      mbar_init(&ds_full[b2], 256);
    }
    mbar_init(acc_full, 1);
    mbar_init(stage_full, 1);
    for (int s = 0; s < IS; ++s) {
      mbar_init(&item_full[s], 1);
      mbar_init(&item_empty[s], kItemReaders);
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
  // Set-up done; the previous kernel's results must be visible from here on.
  grid_dep_wait();

  auto read_item = [&](int k, int& item) {
    if (!mbar_wait(&item_full[k % IS], (k / IS) & 1, abort_flag, kSiteBItem)) return false;
    item = item_slot[k % IS];
    return true;
  };
  auto decode = [&](int item) {
    return dq_item<MODE, PACKED>(item, Hq, group, nqb, tail_heads, n_items, geom, win);
  };

  if (warp == 8) {
    if (lane == 0) {
      // -------------------------------------------------------- producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      uint32_t gk = 0, gv = 0;   // K and V loads issued (ring positions)
      int qd_loads = 0;
      int item = blockIdx.x, next = -1;
      bool ok = true;
      // One ring per operand: K_j, then V_j, each into its own ring.
      auto load = [&](const DqItem& it, int jj, bool is_v, uint32_t idx) {
        const int ns = is_v ? VS : KS;
        const int s = idx % ns;
        const uint32_t round = idx / ns;
        uint64_t* full = is_v ? &v_full[s] : &k_full[s];
        uint64_t* empty = is_v ? &v_empty[s] : &k_empty[s];
        if (round > 0 && !mbar_wait(empty, (round - 1) & 1u, abort_flag, kSiteBLoadEmpty))
          return false;
        mbar_expect_tx(full, C::kTile);
        uint8_t* dst = smem + (is_v ? C::kVOff : C::kKOff) + s * C::kTile;
#pragma unroll
        for (int a = 0; a < D / 64; ++a)
          tma_load_3d(dst + a * 16384, is_v ? &tm_v : &tm_k, full, a * 64,
                      it.sp.k0 + (it.j_lo + jj) * 128, it.zkv);
        return true;
      };
      for (int k = 0; ok; ++k) {
        DqItem it;
        while (item < n_items) {   // skip numbers past a packed sequence's rows
          it = decode(item);
          if (it.n >= 0) break;
          item = next >= 0 ? next : gridDim.x + atomicAdd(sched, 1);
          next = -1;
        }
        const bool done = item >= n_items;
        const int slot = k % IS;
        if (k >= IS && !mbar_wait(&item_empty[slot], ((k / IS) - 1) & 1, abort_flag, kSiteBItem)) {
          ok = false;
          break;
        }
        item_slot[slot] = done ? -1 : item;
        mbar_arrive(&item_full[slot]);
        if (done) break;
        if (next < 0) next = gridDim.x + atomicAdd(sched, 1);
        if (it.n > 0) {
          if (qd_loads > 0 && !mbar_wait(qd_empty, (qd_loads - 1) & 1, abort_flag, kSiteBLoadEmpty)) {
            ok = false;
            break;
          }
          mbar_expect_tx(qd_full, 2 * C::kTile);
#pragma unroll
          for (int a = 0; a < D / 64; ++a) {
            tma_load_3d(smem + C::kQOff + a * 16384, &tm_q, qd_full, a * 64,
                        it.sp.q0 + it.i * 128, it.zq);
            tma_load_3d(smem + C::kDOOff + a * 16384, &tm_do, qd_full, a * 64,
                        it.sp.q0 + it.i * 128, it.zq);
          }
          ++qd_loads;
          for (int jj = 0; jj < it.n; ++jj) {
            if (!load(it, jj, false, gk)) { ok = false; break; }
            ++gk;
            if (!load(it, jj, true, gv)) { ok = false; break; }
            ++gv;
          }
        }
        item = next;
        next = -1;
      }
      // Let every copy this thread started land before the CTA can exit.
      if (qd_loads > 0) mbar_wait_drain(qd_full, (qd_loads - 1) & 1);
      for (uint32_t x = gk > static_cast<uint32_t>(KS) ? gk - KS : 0u; x < gk; ++x)
        mbar_wait_drain(&k_full[x % KS], (x / KS) & 1u);
      for (uint32_t x = gv > static_cast<uint32_t>(VS) ? gv - VS : 0u; x < gv; ++x)
        mbar_wait_drain(&v_full[x % VS], (x / VS) & 1u);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // -------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, 0, 1);
      auto kslot = [&](uint32_t x) { return sbase + C::kKOff + (x % KS) * C::kTile; };
      auto vslot = [&](uint32_t x) { return sbase + C::kVOff + (x % VS) * C::kTile; };
      auto k_wait = [&](uint32_t x) {
        return mbar_wait(&k_full[x % KS], (x / KS) & 1u, abort_flag, kSiteBKV);
      };
      auto v_wait = [&](uint32_t x) {
        return mbar_wait(&v_full[x % VS], (x / VS) & 1u, abort_flag, kSiteBKV);
      };
      // dP / dS of step g live in TMEM columns [128, 256) (even g) or [384, 512) (odd g).
      auto dp_col = [&](uint32_t x) { return (x & 1) ? 384u : 128u; };
      auto mma_tile_kk = [&](uint32_t dst, uint32_t a, uint32_t bt) {
        const SDesc ad = sdesc_sw128_split(a, 16, 1024), bd = sdesc_sw128_split(bt, 16, 1024);
        mma_ss_w<0>(dst, ad.lo, ad.hi, bd.lo, bd.hi, kIdescSS);
#pragma unroll
        for (int kk = 1; kk < D / 16; ++kk) {
          const uint32_t o = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          mma_ss_w<1>(dst, ad.lo + o, ad.hi, bd.lo + o, bd.hi, kIdescSS);
        }
      };
      uint32_t g = 0;            // steps over all items; K and V ring positions match it
      int qd_loads = 0;
      bool ok = true, any = false;
      for (int k = 0; ok; ++k) {
        int item;
        if (!read_item(k, item)) { ok = false; break; }
        mbar_arrive(&item_empty[k % IS]);
        if (item < 0) break;
        const DqItem it = decode(item);
        const int n = it.n;
        if (n <= 0) continue;
        if (!mbar_wait(qd_full, qd_loads & 1, abort_flag, kSiteBLoadFull) || !k_wait(g)) {
          ok = false;
          break;
        }
        ++qd_loads;
        any = true;
        tc_fence_after();
        mma_tile_kk(tmem + 0, sbase + C::kQOff, kslot(g));            // S(0) = Q K_0^T
        tc_commit(s_full);
        if (!v_wait(g)) { ok = false; break; }
        tc_fence_after();
        mma_tile_kk(tmem + dp_col(g), sbase + C::kDOOff, vslot(g));   // dP(0) = dO V_0^T
        tc_commit(&dp_full[g & 1]);
        tc_commit(&v_empty[g % VS]);
        if (n == 1) tc_commit(qd_empty);
        for (int jj = 0; ok && jj < n; ++jj, ++g) {
          const bool more = jj + 1 < n;
          if (more) {
            // S(j+1) once S(j) is in registers; dP(j+1) into the buffer dQ(j-1) has read.
            if (!mbar_wait(s_free, g & 1u, abort_flag, kSiteBSFree) || !k_wait(g + 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            mma_tile_kk(tmem + 0, sbase + C::kQOff, kslot(g + 1));
            tc_commit(s_full);
            if (!v_wait(g + 1)) { ok = false; break; }
            tc_fence_after();
            mma_tile_kk(tmem + dp_col(g + 1), sbase + C::kDOOff, vslot(g + 1));
            tc_commit(&dp_full[(g + 1) & 1]);
            tc_commit(&v_empty[(g + 1) % VS]);
            if (jj + 2 == n) tc_commit(qd_empty);
          }
          if (!mbar_wait(&ds_full[g & 1], (g >> 1) & 1u, abort_flag, kSiteBDS)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const SDesc kbd = sdesc_sw128_split(kslot(g), 16384, 1024);   // dQ += dS K_j
          const uint32_t dsc = tmem + dp_col(g);
          mma_ts_w<-1>(tmem + 256, dsc + split_col(0), kbd.lo, kbd.hi, kIdescAcc,
                       jj > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < 8; ++kk)
            mma_ts_w<1>(tmem + 256, dsc + split_col(kk), kbd.lo + kk * 128, kbd.hi, kIdescAcc);
          // The last key block's slot is released by the store thread instead.
          if (more) tc_commit(&k_empty[g % KS]);
        }
        if (ok) tc_commit(acc_full);
      }
      if (any) {                             // nothing to drain when nothing was issued
        tc_commit(mma_done);
        mbar_wait_drain(mma_done, 0);
      }
    }
    __syncwarp();
  } else if (warp == 10) {
    if (lane == 0) {
      // -------------------------------------------------------- output store
      tma_prefetch_desc(&tm_dq);
      uint32_t g = 0;
      int staged = 0;
      for (int k = 0;; ++k) {
        int item;
        if (!read_item(k, item)) break;
        mbar_arrive(&item_empty[k % IS]);
        if (item < 0) break;
        const DqItem it = decode(item);
        if (it.n <= 0) continue;
        g += it.n;
        if (!mbar_wait(stage_full, staged & 1, abort_flag, kSiteBStage)) break;
        ++staged;
        const int slot = (g - 1) % KS;
        if (!PACKED || it.i * 128 + 128 <= it.sp.nq) {
          uint8_t* tile = smem + C::kKOff + slot * C::kTile;
#pragma unroll
          for (int a = 0; a < D / 64; ++a)
            tma_store_3d(&tm_dq, tile + a * 16384, a * 64, it.sp.q0 + it.i * 128, it.zq);
          bulk_commit_group();
          bulk_wait_read_all();
        }
        mbar_arrive(&k_empty[slot]);
      }
      bulk_wait_read_all();
    }
    __syncwarp();
  } else if (warp < 8) {
    // ---------------------------------------------------------- compute
    const int h = warp >> 2;                         // column half of the step tile
    const int quad = warp & 3;
    const int t = quad * 32 + lane;                  // query row within the block
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t t_s = tmem + lane_base + 64 * h;
    const uint32_t t_dp0 = tmem + lane_base + 128 + 64 * h;  // dP half of buffer 0; dS into +0..32
    const int c_base = 64 * h;
    uint32_t g = 0;
    int acc_items = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int item = -1;
      if (!read_item(k, item)) ok = false;
      __syncwarp();
      if (lane == 0) mbar_arrive(&item_empty[k % IS]);
      // All compute threads agree before going on, so that every named
      // barrier below is reached by all of them or by none.
      ok = named_barrier_and(1, 256, ok);
      if (!ok || item < 0) break;
      const DqItem it = decode(item);
      const int i = it.i, n = it.n, Nq = it.sp.nq, Nk = it.sp.nk;
      KeyWindow w = win;
      w.off = Nk - Nq;
      const int row = i * 128 + t;
      const int r_first = i * 128, r_last = min(i * 128 + 127, Nq - 1);
      // Visible keys of this row: [k_lo, k_hi].
      const int k_lo = (MODE == kMaskGeneral) ? max(0, w.lo(row)) : 0;
      const int k_hi = (MODE == kMaskGeneral) ? min(Nk - 1, w.hi(row))
                                              : ((MODE == kMaskCausal) ? min(row, Nk - 1) : Nk - 1);
      const size_t ws = static_cast<size_t>(it.bh) * Npad + row;   // row < Npad always
      const float nLr = n > 0 ? Lws[ws] : 0.f;                     // -lse*log2e; -inf on padding rows
      const float nDr = n > 0 ? Dws[ws] : 0.f;                     // -rowsum(dO*O)
      for (int jj = 0; ok && jj < n; ++jj, ++g) {
        if (!mbar_wait(s_full, g & 1u, abort_flag, kSiteBS)) { ok = false; break; }
        tc_fence_after();
        uint32_t r0[32], r1[32];
        tmem_ld32(t_s, r0);
        tmem_ld32(t_s + 32, r1);
        tmem_ld_wait(r0);
        reg_fence(r1);
        tc_fence_before();
        mbar_arrive(s_free);
        const int kb = (it.j_lo + jj) * 128;
        // Masked tiles: those crossing an edge of some row's visible keys,
        // including the ragged last tile (keys past Nk are zero rows from the
        // TMA fill; P = 0 there keeps an extreme lse from making 0 * inf).
        bool edge;
        if (MODE == kMaskNone) edge = kb + 127 >= Nk;
        else if (MODE == kMaskCausal) edge = kb + 127 > min(r_first, Nk - 1) || kb + 127 >= Nk;
        else edge = kb < (r_last >= 0 ? w.lo(r_last) : 0) || kb + 127 > min(Nk - 1, w.hi(r_first));
        const int c_lo = k_lo - kb, c_hi = k_hi - kb;   // keep columns [c_lo, c_hi]
        const float2 sc2 = make_float2(scale_log2, scale_log2);
        const float2 nl2 = make_float2(nLr, nLr);
        float pf[64];                                   // P in fp32
        auto p_block = [&](const uint32_t (&r)[32], int c0) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = c_base + c0 + 2 * e;
            float p0, p1;
            if constexpr (SOFTCAP) {
              // dS needs P * (1 - t^2): the chain rule through c * tanh(z / c).
              const float t0 = softcap_tanh(u2f(r[2 * e]), cap);
              const float t1 = softcap_tanh(u2f(r[2 * e + 1]), cap);
              p0 = fast_exp2(fmaf(cap.out, t0, nLr)) * fmaf(-t0, t0, 1.f);
              p1 = fast_exp2(fmaf(cap.out, t1, nLr)) * fmaf(-t1, t1, 1.f);
            } else {
              const float2 x = ffma2(make_float2(u2f(r[2 * e]), u2f(r[2 * e + 1])), sc2, nl2);
              p0 = fast_exp2(x.x);
              p1 = fast_exp2(x.y);
            }
            if (edge) {
              if (MODE == kMaskGeneral) {
                if (c < c_lo || c > c_hi) p0 = 0.f;
                if (c + 1 < c_lo || c + 1 > c_hi) p1 = 0.f;
              } else {                                  // k_lo = 0: one-sided
                if (c > c_hi) p0 = 0.f;
                if (c + 1 > c_hi) p1 = 0.f;
              }
            }
            pf[c0 + 2 * e] = p0;
            pf[c0 + 2 * e + 1] = p1;
          }
        };
        p_block(r0, 0);
        p_block(r1, 32);

        // dP(j) and dS(j) use buffer g & 1 (TMEM columns 128.. or 384..).
        const uint32_t t_dp = t_dp0 + (g & 1) * 256;
        if (!mbar_wait(&dp_full[g & 1], (g >> 1) & 1u, abort_flag, kSiteBDP)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t d0[32], d1[32];
        tmem_ld32(t_dp, d0);
        tmem_ld32(t_dp + 32, d1);
        tmem_ld_wait(d0);
        reg_fence(d1);
        uint32_t ds[32];
        const float2 nd2 = make_float2(nDr, nDr);
        auto nd = [&](int) { return nd2; };
        ds_block(&pf[0], d0, ds, nd);
        ds_block(&pf[32], d1, ds + 16, nd);
        tmem_st32(t_dp, ds);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&ds_full[g & 1]);
      }
      if (ok && n > 0) ok = mbar_wait(acc_full, acc_items & 1, abort_flag, kSiteBAcc);
      // Every compute thread gets here once per item; the epilogue runs only
      // if all of them completed their waits.
      ok = named_barrier_and(1, 256, ok);
      if (!ok) break;
      const bool valid = row < Nq;
      const long long o_z = PACKED ? geom.o_z : static_cast<long long>(Nq) * D;
      const long long o_row = PACKED ? geom.o_row : D;
      __nv_bfloat16* dst = dq + it.zq * o_z + (it.sp.q0 + (valid ? row : 0)) * o_row;
      if (n > 0) {
        ++acc_items;
        tc_fence_after();
        // A full tile goes through shared memory (the K ring slot of the last
        // key block) and a TMA store; each warpgroup stages its own 64-column
        // half. A packed tile that runs past its sequence is written row by row.
        if (!PACKED || i * 128 + 128 <= Nq) {
          uint8_t* tile = smem + C::kKOff + ((g - 1) % KS) * C::kTile;
          if (h == 0)
            stage_acc_row<D, 0, D / 64>(tmem + lane_base + 256, tile, t, scale);
          else
            stage_acc_row<D, D / 64, D / 32>(tmem + lane_base + 256, tile, t, scale);
          fence_proxy_async_smem();
        } else if (h == 0) {
          store_acc_row<D, 0, D / 64>(tmem + lane_base + 256, dst, scale, valid);
        } else {
          store_acc_row<D, D / 64, D / 32>(tmem + lane_base + 256, dst, scale, valid);
        }
        tc_fence_before();
        named_barrier_sync(1, 256);
        if (threadIdx.x == 0) mbar_arrive(stage_full);
      } else if (valid) {
        // This query block sees no key: its gradient is zero.
        uint4* p = reinterpret_cast<uint4*>(dst) + h * (D / 16);
#pragma unroll
        for (int c = 0; c < D / 16; ++c) p[c] = make_uint4(0u, 0u, 0u, 0u);
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
