// mlra_merge.cuh -- merging the partial softmax states of a split sequence, shared by the combine
// kernel and the step-3 product kernel that merges while it stages its input.
//
// A part p of (sequence, head, branch) holds m_p (running maximum of the scaled scores, log2
// units), l_p = sum_j 2^(s_j - m_p) and the unnormalised output o_p = sum_j 2^(s_j - m_p) c_j.
// The merged state is m* = max_p m_p, l* = sum_p 2^(m_p - m*) l_p, o* = sum_p 2^(m_p - m*) o_p,
// after which out = gamma o* / l* and lse = (m* + log2 l*) ln 2.  The fold below visits the parts
// one by one with a running maximum, which gives the same sums.
#pragma once
#include <cstdint>
#include <math_constants.h>

namespace mlra {

constexpr int kMergeUnroll = 8;  // parts whose loads are issued together (one round trip)

struct MergeState {
  float m, l;
  float4 acc;
};

__device__ __forceinline__ MergeState merge_empty() {
  return MergeState{-CUDART_INF_F, 0.f, make_float4(0.f, 0.f, 0.f, 0.f)};
}

// Folds one part (or another partial merge) into st.  A state with m = -inf carries no weight.
__device__ __forceinline__ void merge_into(MergeState& st, float m_p, float l_p, float4 o_p) {
  const float mn = fmaxf(st.m, m_p);
  const float a = st.m == -CUDART_INF_F ? 0.f : exp2f(st.m - mn);
  const float w = m_p == -CUDART_INF_F ? 0.f : exp2f(m_p - mn);
  st.l = st.l * a + l_p * w;
  st.acc.x = st.acc.x * a + o_p.x * w;
  st.acc.y = st.acc.y * a + o_p.y * w;
  st.acc.z = st.acc.z * a + o_p.z * w;
  st.acc.w = st.acc.w * a + o_p.w * w;
  st.m = mn;
}

// Parts g, g+G, ... < np of (head h, branch b) at padded latent column k (4 columns), stored in
// slots slot0 + p of part_ml [slots, H, B, 2] and part_o [slots, H, dck].  The partials were
// written by other SMs during the current or the previous launch: read them through L2.
__device__ __forceinline__ MergeState fold_parts(const float* part_ml, const float* part_o, int H,
                                                 int B, int dck, int64_t slot0, int np, int g,
                                                 int G, int h, int b, int k) {
  MergeState st = merge_empty();
  for (int p0 = g; p0 < np; p0 += G * kMergeUnroll) {
    float2 ml[kMergeUnroll];
    float4 v[kMergeUnroll];
#pragma unroll
    for (int u = 0; u < kMergeUnroll; ++u) {
      const int pp = p0 + u * G;
      if (pp < np) {
        const int64_t row = (slot0 + pp) * H + h;
        ml[u] = __ldcg(reinterpret_cast<const float2*>(part_ml + (row * B + b) * 2));
        v[u] = __ldcg(reinterpret_cast<const float4*>(part_o + row * dck + k));
      }
    }
#pragma unroll
    for (int u = 0; u < kMergeUnroll; ++u)
      if (p0 + u * G < np) merge_into(st, ml[u].x, ml[u].y, v[u]);
  }
  return st;
}

// Writes gamma * acc / l to dst[0 .. min(4, ncols)) (float4 when aligned).
__device__ __forceinline__ void store_merged(float* dst, const MergeState& st, float gamma,
                                             int ncols) {
  const float sc = gamma / st.l;
  const float r[4] = {st.acc.x * sc, st.acc.y * sc, st.acc.z * sc, st.acc.w * sc};
  if (ncols >= 4 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
    *reinterpret_cast<float4*>(dst) = make_float4(r[0], r[1], r[2], r[3]);
  } else {
    for (int j = 0; j < 4 && j < ncols; ++j) dst[j] = r[j];
  }
}

__device__ __forceinline__ float merged_lse(const MergeState& st) {
  return (st.m + log2f(st.l)) * 0.69314718055994531f;
}

}  // namespace mlra
