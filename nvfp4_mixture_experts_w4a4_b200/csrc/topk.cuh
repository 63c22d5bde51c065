// Warp top-k over one token's router logits, shared by moe_route and the small-batch
// prologue so both select and weight experts identically.
//
// Lane l holds logits l, l+32, ... (PER_LANE slots, E <= 32*PER_LANE) as 64-bit keys: the
// high word is the logit mapped to an unsigned integer with the same order (after -0 is
// turned into +0, so the two zeros tie), the low word is 0xFFFF - index, so among equal
// logits the lower index has the larger key.  Each lane keeps its best remaining key; a
// round is a warp max over those and only the winning lane advances its own best.
// Integer compares make the selection exact; the softmax over the k selected logits
// (relative to the largest) is fp32.
#pragma once

#include "common.cuh"

namespace nvfp4moe {

__device__ __forceinline__ uint64_t topk_key(float v, int idx) {
  uint32_t u = __float_as_uint(v + 0.0f);  // -0 + +0 = +0 under round-to-nearest
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (uint64_t(u) << 32) | uint32_t(0xFFFF - idx);
}

__device__ __forceinline__ int topk_key_index(uint64_t key) { return 0xFFFF - int(uint32_t(key) & 0xFFFFu); }

// The logit a key was built from (the order-preserving map inverted; -0 comes back as +0).
__device__ __forceinline__ float topk_key_value(uint64_t key) {
  const uint32_t u = uint32_t(key >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// Selects the top k (k <= 32) of the E logits the calling warp holds, lane l holding logits
// l, l+32, ... in lg[] (slots at or past E are ignored).  Lane j < k returns the j-th expert in
// *id and its softmax weight in *w.  Each lane first finds its two largest keys.  A round takes
// the warp maximum of the lanes' current best keys with two hardware reductions (the logit
// word, then the index word among the lanes that hold that logit, which picks the lower expert
// index); the lane that held the winner moves on to its second key, and only on a further win
// rescans its keys for the largest one below the key just taken (keys are unique, so "below"
// excludes exactly the keys already taken).  A lane rarely holds more than two of the k
// winners, so the rescans are rare and most rounds cost two reductions.
template <int PER_LANE>
__device__ __forceinline__ void warp_topk_regs(const float (&lg)[PER_LANE], int E, int k, int* id, float* w) {
  const int lane = threadIdx.x & 31;
  uint64_t key[PER_LANE];
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? topk_key(lg[i], e) : 0ull;  // 0 marks an absent slot (real keys are > 0)
  }
  uint64_t m1 = 0, m2 = 0;  // this lane's largest and second largest key
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const uint64_t v = key[i];
    const bool top = v > m1;
    m2 = top ? m1 : (v > m2 ? v : m2);
    m1 = top ? v : m1;
  }
  bool second = true;  // m2 is still this lane's next key
  uint64_t sel = 0;    // lane j keeps the j-th selected key
  for (int j = 0; j < k; ++j) {
    const uint32_t hi = uint32_t(m1 >> 32), lo = uint32_t(m1);
    const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t mlo = __reduce_max_sync(0xffffffffu, hi == mhi ? lo : 0u);
    const uint64_t best = (uint64_t(mhi) << 32) | mlo;
    if (lane == j) sel = best;
    if (best == m1) {  // this lane held the winner
      if (second) {
        m1 = m2;
        second = false;
      } else {
        uint64_t nm = 0;
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) nm = (key[i] < best && key[i] > nm) ? key[i] : nm;
        m1 = nm;
      }
    }
  }
  const int bi = topk_key_index(sel);
  const float sel_v = lane < k ? topk_key_value(sel) : 0.0f;
  const float l0 = __shfl_sync(0xffffffffu, sel_v, 0);
  const float ex = lane < k ? expf(sel_v - l0) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  *id = bi;
  *w = ex / sum;
}

// The same selection over l[0..E) in global memory.
template <int PER_LANE>
__device__ __forceinline__ void warp_topk(const float* __restrict__ l, int E, int k, int* id, float* w) {
  const int lane = threadIdx.x & 31;
  float lg[PER_LANE];
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const int e = lane + 32 * i;
    lg[i] = e < E ? l[e] : 0.0f;
  }
  warp_topk_regs<PER_LANE>(lg, E, k, id, w);
}

}  // namespace nvfp4moe
