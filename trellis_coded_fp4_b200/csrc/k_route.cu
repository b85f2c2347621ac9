// k_route.cu -- MoE router: top-k experts per token and softmax weights over the selected logits.
//
// The routed-MoE workloads use "top-k selection and softmax weights": the k largest logits (ties
// to the lower expert index) and w_j = exp(l_j - l_max) / sum_i exp(l_i - l_max) over the k
// selected logits, in fp32. One warp per token; each lane holds E/32 logits; k rounds of a warp
// arg-max that orders by (value descending, index ascending).
#include "tcf4_internal.h"

namespace tcf4 {

__global__ void __launch_bounds__(256) k_route(const float *__restrict__ logits, int T, int E, int k,
                                               int32_t *__restrict__ ids, float *__restrict__ wts) {
  grid_dep_wait();  // the logits come from the preceding kernel
  grid_dep_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  constexpr int kPer = kMaxExperts / 32;
  float v[kPer];
#pragma unroll
  for (int i = 0; i < kPer; i++) {
    const int e = i * 32 + lane;
    v[i] = e < E ? logits[(size_t)t * E + e] : -INFINITY;
  }
  bool used[kPer];
#pragma unroll
  for (int i = 0; i < kPer; i++) used[i] = false;
  float sel_v[kMaxTopK];
  int sel_e[kMaxTopK];
  for (int r = 0; r < k; r++) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPer; i++) {
      const int e = i * 32 + lane;
      if (e < E && !used[i] && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    sel_v[r] = bv;
    sel_e[r] = be;
#pragma unroll
    for (int i = 0; i < kPer; i++)
      if (i * 32 + lane == be) used[i] = true;  // remove the winner (its lane owns it)
  }
  if (lane == 0) {
    const float mx = sel_v[0];
    float den = 0.f;
    for (int r = 0; r < k; r++) den += expf(sel_v[r] - mx);
    for (int r = 0; r < k; r++) {
      ids[t * k + r] = sel_e[r];
      wts[t * k + r] = expf(sel_v[r] - mx) / den;
    }
  }
}

cudaError_t launch_route(const float *logits, int T, int E, int k, int32_t *ids, float *wts, cudaStream_t s) {
  return launch_dependent(k_route, dim3((T + 7) / 8), dim3(256), 0, s, logits, T, E, k, ids, wts);
}

}  // namespace tcf4
