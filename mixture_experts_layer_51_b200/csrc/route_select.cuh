// TopK + gating softmax (or the expert-choice affinities) of tokens whose
// logits sit in shared memory, shared by the router kernels.
//
// Pages: "How do Mixture of Expert Models Work?", "The Math Behind MoEs"
// (G(x) = Softmax(TopK(x . W_g)): the k largest logits, then the softmax over
// them); "[Paper Club] Upcycling Large Language Models into Mixture of
// Experts" (Switch order: the softmax over all experts first, so the selected
// probabilities no longer sum to one, with an optional scale of the output).
//
// P threads cooperate on one token (P a power of two, the P lanes adjacent
// in one warp).  Each keeps the sorted top-(k+1) list of a contiguous range
// of experts (a compare-and-swap chain), then the lists are merged in a
// butterfly in which the lower half's list goes first, so equal logits keep
// the lower expert first -- the stable descending order -- and every thread
// ends with the same list.
#pragma once

#include <math.h>

#include "moe_internal.cuh"

namespace moe {

// (v, ei) goes before (w, ej): a larger value, or an equal value and a lower
// expert -- the stable descending order.  (Bitwise operators: with the
// short-circuit ones the selection below ran 1.7 times slower.)
__device__ __forceinline__ bool ranks_before(float v, int ei, float w, int ej) {
  return (v > w) | ((v == w) & (ei < ej));
}

// Inserts (v, ei) into a list sorted in that order (ei < 0: nothing to
// insert).  An unfilled slot (index < 0) always takes the entry, so -inf
// logits are still ranked in expert order.  An entry pushed down the list
// is compared by value and expert, so it stays in front of an equal logit
// of a higher expert.
template <int KM>
__device__ __forceinline__ void insert_sorted(float (&tv)[KM], int (&ti)[KM], float v, int ei) {
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    const bool take = (ei >= 0) & ((ti[j] < 0) | ranks_before(v, ei, tv[j], ti[j]));
    const float tvj = tv[j];
    const int tij = ti[j];
    tv[j] = take ? v : tvj;
    ti[j] = take ? ei : tij;
    v = take ? tvj : v;
    ei = take ? tij : ei;
  }
}

// Merges two lists sorted as insert_sorted keeps them into the first: the
// KM leading entries of their union, in the same order; a real entry goes
// before an unfilled one.  Each step takes the larger head and shifts
// that list by one -- only the entries that may still be taken move.
template <int KM>
__device__ __forceinline__ void merge_sorted(float (&av)[KM], int (&ai)[KM], float (&bv)[KM],
                                             int (&bi)[KM]) {
  float ov[KM];
  int oi[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    const bool ta = (ai[0] >= 0) & ((bi[0] < 0) | ranks_before(av[0], ai[0], bv[0], bi[0]));
    ov[j] = ta ? av[0] : bv[0];
    oi[j] = ta ? ai[0] : bi[0];
    // Fixed bounds, so the lists stay in registers; the entries past
    // KM - 1 - j are never taken again, so shifting them as well is harmless.
#pragma unroll
    for (int i = 0; i + 1 < KM; ++i) {
      av[i] = ta ? av[i + 1] : av[i];
      ai[i] = ta ? ai[i + 1] : ai[i];
      bv[i] = ta ? bv[i] : bv[i + 1];
      bi[i] = ta ? bi[i] : bi[i + 1];
    }
  }
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    av[j] = ov[j];
    ai[j] = oi[j];
  }
}

// One token's selection.  lrow: its E logits (bias included); p: this
// thread's place among the token's P threads; t: the token (written only if
// `valid`).  Writes idx/gate [T, k] (slot order = descending logit), margin
// [T] (k-th minus (k+1)-th logit, +inf when k == E; nullable) and, when
// idx_s is given, the k selected experts to idx_s[0..k-1] (shared memory,
// written by p == 0).  All P threads of a token must call it together; the
// calling warp must be converged.
template <int KM>
__device__ __forceinline__ void select_token(const float* lrow, int E, int k, int P, int p,
                                             int t, bool valid, int gating, float gate_scale,
                                             int32_t* __restrict__ idx, float* __restrict__ gate,
                                             float* __restrict__ margin, int* idx_s) {
  float tv[KM];
  int ti[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    tv[j] = -INFINITY;
    ti[j] = -1;
  }
  {
    const int per = (E + P - 1) / P;
    const int e_lo = min(E, p * per), e_hi = min(E, e_lo + per);
    for (int e = e_lo; e < e_hi; ++e) insert_sorted<KM>(tv, ti, lrow[e], e);
  }
  for (int o = 1; o < P; o <<= 1) {
    float pv[KM];
    int pi[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      pv[j] = __shfl_xor_sync(0xffffffffu, tv[j], o);
      pi[j] = __shfl_xor_sync(0xffffffffu, ti[j], o);
    }
    if (p & o) {
      // The partner holds the lower experts: its list goes first.
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        const float v = tv[j];
        const int ei = ti[j];
        tv[j] = pv[j];
        ti[j] = pi[j];
        pv[j] = v;
        pi[j] = ei;
      }
    }
    merge_sorted<KM>(tv, ti, pv, pi);
  }
  const float m = tv[0];  // the largest logit
  float denom = 0.f;
  if (gating == MOE_GATE_SOFTMAX_TOPK) {
    // Switch order: the softmax denominator over all E logits.
    for (int e = p; e < E; e += P) denom += expf(lrow[e] - m);
    for (int o = P / 2; o > 0; o >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, o);
  } else {
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (j < k) denom += expf(tv[j] - m);
  }
  if (!valid) return;
  const float inv = gate_scale / denom;
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    if (j < k && j % P == p) {
      idx[(int64_t)t * k + j] = ti[j];
      gate[(int64_t)t * k + j] = expf(tv[j] - m) * inv;
    }
  }
  if (idx_s && p == 0) {
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (j < k) idx_s[j] = ti[j];
  }
  if (margin) {
    // slot k-1 minus slot k (every gap computed, one kept: no dynamic
    // index into the list)
    float mg = INFINITY;
#pragma unroll
    for (int j = 1; j < KM; ++j) {
      const float gap = tv[j - 1] - tv[j];
      mg = (j == k && k < E) ? gap : mg;
    }
    if (p == 0) margin[t] = mg;
  }
}

// Expert-choice affinities of one token: the softmax over all E logits,
// combined over its P threads with a fixed butterfly.  Returns the maximum
// and the reciprocal of the sum (every lane of the token gets the same).
__device__ __forceinline__ void softmax_stats(const float* lrow, int E, int P, int p, float& m,
                                              float& inv) {
  m = -INFINITY;
  for (int e = p; e < E; e += P) m = fmaxf(m, lrow[e]);
  for (int o = P / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float sum = 0.f;
  for (int e = p; e < E; e += P) sum += expf(lrow[e] - m);
  for (int o = P / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  inv = 1.f / sum;
}

}  // namespace moe
