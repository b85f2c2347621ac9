// k_route.cu -- MoE router: top-k experts per token and softmax weights over the selected logits.
//
// The routed-MoE workloads use "top-k selection and softmax weights": the k largest logits (ties
// to the lower expert index) and w_j = exp(l_j - l_max) / sum_i exp(l_i - l_max) over the k
// selected logits, in fp32. One warp per token; each lane holds E/32 logits; k rounds of a warp
// arg-max that orders by (key descending, index ascending), where the key is the logit's bit
// pattern made order-preserving as a signed integer, -0 counted as +0 and NaN below every number
// (so k valid ids always come out). In the softmax a NaN logit counts as -inf; when the largest
// selected logit is -inf every weight is 0, and when it is +inf the +inf logits share the weight.
#include <climits>

#include "tcf4_internal.h"

namespace tcf4 {

// Order-preserving integer key of a logit: larger logit, larger key; -0 and +0 share a key; every
// NaN gets the smallest key (below -inf).
__device__ __forceinline__ int route_key(float v) {
  if (v != v) return INT_MIN;
  const int b = __float_as_int(v + 0.0f);  // -0 + 0 = +0
  return b >= 0 ? b : b ^ 0x7fffffff;
}
// The logit a key stands for (NaN's key reads as -inf).
__device__ __forceinline__ float key_logit(int key) {
  if (key == INT_MIN) return -INFINITY;
  return __int_as_float(key >= 0 ? key : key ^ 0x7fffffff);
}

__global__ void __launch_bounds__(256) k_route(const float *__restrict__ logits, int T, int E, int k,
                                               int32_t *__restrict__ ids, float *__restrict__ wts) {
  grid_dep_wait();  // the logits come from the preceding kernel
  grid_dep_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  constexpr int kPer = kMaxExperts / 32;
  int key[kPer];
#pragma unroll
  for (int i = 0; i < kPer; i++) {
    const int e = i * 32 + lane;
    key[i] = e < E ? route_key(logits[(size_t)t * E + e]) : INT_MIN;
  }
  bool used[kPer];
#pragma unroll
  for (int i = 0; i < kPer; i++) used[i] = false;
  int sel_k[kMaxTopK];
  int sel_e[kMaxTopK];
  for (int r = 0; r < k; r++) {
    int bk = INT_MIN;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPer; i++) {
      const int e = i * 32 + lane;
      if (e < E && !used[i] && (key[i] > bk || (key[i] == bk && e < be))) {
        bk = key[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const int ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ok > bk || (ok == bk && oe < be)) {
        bk = ok;
        be = oe;
      }
    }
    sel_k[r] = bk;
    sel_e[r] = be;
#pragma unroll
    for (int i = 0; i < kPer; i++)
      if (i * 32 + lane == be) used[i] = true;  // remove the winner (its lane owns it)
  }
  if (lane == 0) {
    const float mx = key_logit(sel_k[0]);
    float den = 0.f;
    int ninf = 0;
    for (int r = 0; r < k; r++) {
      den += expf(key_logit(sel_k[r]) - mx);
      ninf += key_logit(sel_k[r]) == INFINITY;
    }
    for (int r = 0; r < k; r++) {
      const float l = key_logit(sel_k[r]);
      ids[t * k + r] = sel_e[r];
      wts[t * k + r] = mx == -INFINITY ? 0.f
                       : mx == INFINITY ? (l == INFINITY ? 1.f / (float)ninf : 0.f)
                                        : expf(l - mx) / den;
    }
  }
}

cudaError_t launch_route(const float *logits, int T, int E, int k, int32_t *ids, float *wts, cudaStream_t s) {
  return launch_dependent(k_route, dim3((T + 7) / 8), dim3(256), 0, s, logits, T, E, k, ids, wts);
}

}  // namespace tcf4
