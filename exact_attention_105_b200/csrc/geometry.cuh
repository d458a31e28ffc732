// Where each (sequence, head) of a batch lives in memory, and the softcap
// transform of the scores.
//
// Two batch layouts share one set of kernels:
//   fixed length  Q/O/dO/dQ [B, Hq, N, d], K/V/dK/dV [B, Hkv, N, d], lse [B, Hq, N]
//   packed        Q/O/dO/dQ [total_q, Hq, d], K/V/dK/dV [total_k, Hkv, d],
//                 lse [Hq, total_q]; sequence b is rows cu_q[b] .. cu_q[b+1]
// hysenlabs.com "FlashAttention: exakte Attention-Kernel fuer CUDA und ROCm",
// section "Von 2.0 bis 2.7": release 2.0 names the unpadded functions
// "varlen". The packed layout stores sequences token by token with no padding.
//
// Every tensor map is 3-D (d, rows, z) with strides chosen per layout, so a
// tile of 128 rows of one head is the same TMA box in both: rows of the
// fixed layout are consecutive within a head (z = b * H + h), and rows of the
// packed layout are H * d elements apart (z = h, row = cu[b] + r).
//
// Softcapping, release 2.6 on the same page: the scaled logit z = scale * s
// becomes c * tanh(z / c). In log2 units, with t = tanh(z / c),
//     c * log2(e) * t,   t = 1 - 2 / (2^(2 z log2(e) / c) + 1),
// which costs two SFU operations (ex2, rcp) per score on top of the softmax
// exponential. The form is exact for every finite z: a huge exponent gives
// rcp(inf) = 0 and t = 1, a very negative one gives t = -1.
#pragma once

#include "sm100.cuh"

namespace attn {

struct SeqGeom {
  const int* cu_q;        // [B + 1] row offsets of the packed layout, or nullptr (fixed)
  const int* cu_k;
  int Nq, Nk;             // fixed lengths; for the packed layout the longest sequence
  int total_q, total_k;   // rows of the packed tensors
  long long o_z, o_row;   // element strides of Q-side rows (Q, O, dO, dQ): per z, per row
  long long kv_z, kv_row; // element strides of K-side rows (K, V, dK, dV)
  long long lse_z;        // lse elements per z
};

struct SeqSpan {
  int q0, nq, k0, nk;     // first row and length of the sequence's queries and keys
};

// Rows of sequence b. Packed offsets that are inconsistent (negative, past
// the tensor, decreasing, or longer than the maximum the grid was sized for)
// are clipped into range, so no store can leave the tensors, and the status
// word records kDevBadOffsets for attn_check_status().
template <bool PACKED>
__device__ __forceinline__ SeqSpan seq_span(const SeqGeom& g, int b) {
  if constexpr (!PACKED) return SeqSpan{0, g.Nq, 0, g.Nk};
  int a = g.cu_q[b], e = g.cu_q[b + 1];
  int c = g.cu_k[b], f = g.cu_k[b + 1];
  const bool bad = a < 0 || e < a || e > g.total_q || e - a > g.Nq || c < 0 || f < c ||
                   f > g.total_k || f - c > g.Nk;
  if (bad) {
    if (threadIdx.x == 0) atomicCAS(&g_attn_device_status, 0, kDevBadOffsets);
    a = min(max(a, 0), g.total_q);
    e = min(min(max(e, a), g.total_q), a + g.Nq);
    c = min(max(c, 0), g.total_k);
    f = min(min(max(f, c), g.total_k), c + g.Nk);
  }
  return SeqSpan{a, e - a, c, f - c};
}

// Kernel feature bits (template argument FEAT): softcapped scores, and the
// packed layout (offsets read from cu_q / cu_k). Both run in the general
// mask mode only; the fixed-length fast paths carry neither.
enum : int { kFeatSoftcap = 1, kFeatPacked = 2 };

// Softcap constants: in = 2 * scale * log2(e) / c, out = c * log2(e).
struct Softcap {
  float in, out;
};

__device__ __forceinline__ float fast_rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// tanh(scale * s / c) for a raw score s.
__device__ __forceinline__ float softcap_tanh(float s, const Softcap& sc) {
  return fmaf(-2.0f, fast_rcp(fast_exp2(s * sc.in) + 1.0f), 1.0f);
}

}  // namespace attn
