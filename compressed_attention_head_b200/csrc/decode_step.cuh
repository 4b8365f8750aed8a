// The first launch of a fused decode step: the new token's keys and values
// compressed into the packed caches (append) and the queries prepared for the
// attention partials, by blocks of three roles in one grid. The two roles have
// no data between them (the partials of the second launch read both), so one
// launch replaces the append, the append of the other side, and the prepare.
//
// SpectralQuant README, "Headline Results": decode latency per step over the
// compressed cache; each step appends one token per sequence and attends over
// the whole cache, the new token included.
#pragma once

#include "attention.cuh"
#include "codec.cuh"

namespace sq {

static_assert(append_smem(8) <= prep_smem(kMaxD), "the fused step's shared memory holds every append role");

// Blocks [0, n_app): keys of head i % n_kv, rows of group i / n_kv; [n_app,
// 2 n_app): the same for values; then one prepare block per (KV head, row
// group of prep_rows(G)). 256 threads; shared memory max(append_smem(NV),
// prep_smem(d)).
template <typename T, int NV>
__global__ void __launch_bounds__(256) k_step_prep(const uint8_t* __restrict__ recs_k,
                                                   const uint8_t* __restrict__ recs_v, const T* __restrict__ k_new,
                                                   const T* __restrict__ v_new, const T* __restrict__ q, int batch,
                                                   int n_kv, int d, const int32_t* __restrict__ pos, CacheArgs kc,
                                                   CacheArgs vc, AttnShape s, float scale, float* __restrict__ ws,
                                                   uint32_t* __restrict__ flags, int n_app) {
  extern __shared__ __align__(16) uint8_t ssm[];
  const int bx = blockIdx.x;
  if (bx < 2 * n_app) {
    const int side = bx / n_app, i = bx % n_app;
    append_body<T, NV>(side ? recs_v : recs_k, side ? v_new : k_new, batch, n_kv, d, 1, pos, side ? vc : kc, flags,
                       i % n_kv, i / n_kv, ssm);
  } else {
    const int j = bx - 2 * n_app;
    prepare_body<T>(recs_k, q, s, scale, ws, flags, j % n_kv, (j / n_kv) * prep_rows(s.group), (float*)ssm,
                    threadIdx.x, blockDim.x);
  }
}

}  // namespace sq
