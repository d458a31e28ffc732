// Which keys a query row may see, shared by the forward and backward kernels.
//
// hysenlabs.com "FlashAttention: exakte Attention-Kernel fuer CUDA und ROCm",
// section "Von 2.0 bis 2.7": the causal mask is aligned to the bottom-right
// corner when query and key lengths differ (2.1), and sliding-window
// attention came in 2.3 (`window_size` in the interface section). With
// off = Nk - Nq, query row r sees key j iff
//     r + off - wl <= j <= r + off + wr   and   0 <= j < Nk,
// where an unbounded side is kUnbounded and causal means wr = 0.
//
// Kernels are instantiated for three mask modes:
//   kMaskNone    Nq == Nk, no window, no causal (only a ragged last key tile)
//   kMaskCausal  Nq == Nk, causal, no window (key j <= row)
//   kMaskGeneral any window and/or Nq != Nk
// The first two keep the tuned fast paths and the third uses the bounds above.
#pragma once

namespace attn {

enum MaskMode : int { kMaskNone = 0, kMaskCausal = 1, kMaskGeneral = 2 };
constexpr int kUnbounded = 1 << 30;

struct KeyWindow {
  int off, wl, wr;
  __host__ __device__ int lo(int r) const { return r + off - wl; }  // first visible key
  __host__ __device__ int hi(int r) const { return r + off + wr; }  // last visible key
};

// 128-key tiles [lo, hi] that query rows [r_a, r_b] can see (hi < lo: none).
template <int MODE>
__host__ __device__ inline void kv_tile_range(int r_a, int r_b, int Nk, KeyWindow w, int& lo,
                                              int& hi) {
  const int nkv = (Nk + 127) >> 7;
  if (MODE == kMaskNone) {
    lo = 0;
    hi = nkv - 1;
  } else if (MODE == kMaskCausal) {
    lo = 0;
    hi = min(nkv - 1, r_b >> 7);
  } else {
    const int a = max(0, w.lo(r_a)), b = min(Nk - 1, w.hi(r_b));
    if (a > b) {
      lo = 0;
      hi = -1;
    } else {
      lo = a >> 7;
      hi = b >> 7;
    }
  }
}

// 128-row query blocks [lo, hi] whose rows can see some key of key tile j.
template <int MODE>
__host__ __device__ inline void q_block_range(int j, int Nq, int Nk, KeyWindow w, int& lo,
                                              int& hi) {
  const int nq = (Nq + 127) >> 7;
  if (MODE == kMaskNone) {
    lo = 0;
    hi = nq - 1;
  } else if (MODE == kMaskCausal) {
    lo = j;
    hi = nq - 1;
  } else {
    const int k_a = j * 128, k_b = min(Nk - 1, j * 128 + 127);
    // hi(r) >= k_a  <=>  r >= k_a - off - wr;   lo(r) <= k_b  <=>  r <= k_b - off + wl
    const int a = max(0, k_a - w.off - w.wr), b = min(Nq - 1, k_b - w.off + w.wl);
    if (a > b) {
      lo = 0;
      hi = -1;
    } else {
      lo = a >> 7;
      hi = b >> 7;
    }
  }
}

}  // namespace attn
