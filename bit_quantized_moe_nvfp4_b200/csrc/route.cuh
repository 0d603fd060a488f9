// route.cuh -- arguments of the token-permutation kernel (see route.cu).
#pragma once
#include "common.cuh"

namespace nvfp4 {

constexpr int kMaxExperts = 1024;

struct RouteArgs {
  const int32_t *ids;     // [n_pairs] expert id of pair t*K+k
  int64_t n_pairs;        // T*K
  int E;
  int32_t *counts;        // [E]            (may be null)
  int32_t *offsets;       // [E+1]          (may be null)
  int32_t *perm;          // [n_pairs]      pair indices grouped by expert
  int32_t *inv;           // [n_pairs]      position of each pair in perm, -1 if invalid
  int32_t *flag;          // error flag     (may be null)
  int32_t *active;        // [E]  experts with at least one pair, ascending (may be null)
  int32_t *n_active;      // [1]            (may be null)
  int32_t *tile_prefix;   // [E+1] prefix of ceil(count/tile_n) over active experts (may be null)
  int tile_n;
};

size_t route_smem_bytes(int E);
int launch_route(const RouteArgs &a, cudaStream_t stream, bool pdl);

}  // namespace nvfp4
