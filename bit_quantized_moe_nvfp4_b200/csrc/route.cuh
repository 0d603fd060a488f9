// route.cuh -- arguments of the token-permutation kernel (see route.cu).
#pragma once
#include "common.cuh"

namespace nvfp4 {

constexpr int kMaxExperts = 1024;

// What a routed id means on this device.  Under expert parallelism, rank `rank` of `size`
// owns the experts e in [0, E_global) with e mod size == rank and stores expert e at local
// index e / size; size 1 is the whole layer on one device.
constexpr int kIdForeign = -1;   // a valid expert that another rank owns: skipped, no error
constexpr int kIdBad = -2;       // outside [0, E_global): skipped, error bit kFlagBadId
struct ExpertMap {
  int E_global, size, rank;
  // local index of `id` (>= 0), kIdForeign or kIdBad
  __device__ __forceinline__ int local(int id) const {
    if ((unsigned)id >= (unsigned)E_global) return kIdBad;
    if (size == 1) return id;
    return id % size == rank ? id / size : kIdForeign;
  }
};
inline ExpertMap whole_layer(int64_t E) { return ExpertMap{(int)E, 1, 0}; }

struct RouteArgs {
  const int32_t *ids;     // [n_pairs] expert id of pair t*K+k (global)
  int64_t n_pairs;        // T*K
  int E;                  // experts on this device (local indices 0..E-1)
  ExpertMap map;
  int32_t *counts;        // [E]            (may be null)
  int32_t *offsets;       // [E+1]          (may be null)
  int32_t *perm;          // [n_pairs]      pair indices grouped by expert
  int32_t *inv;           // [n_pairs]      position of each pair in perm, -1 if not local
  int32_t *flag;          // error flag     (may be null)
  int32_t *active;        // [E]  experts with at least one pair, ascending (may be null)
  int32_t *n_active;      // [1]            (may be null)
  int32_t *tile_prefix;   // [E+1] prefix of ceil(count/tile_n) over active experts (may be null)
  int tile_n;
};

size_t route_smem_bytes(int E);
// Pairs per chunk of the many-CTA route; scratch ints it needs (route_scratch_ints).
constexpr int64_t kRouteChunk = 2048;
int64_t route_scratch_ints(int64_t n_pairs, int E);
// The route step: one CTA, or, with scratch of route_scratch_ints(n_pairs, E) int32 and more
// than kRouteChunk pairs, three kernels over many CTAs (the same result).
int launch_route(const RouteArgs &a, cudaStream_t stream, bool pdl, int32_t *scratch = nullptr);

}  // namespace nvfp4
