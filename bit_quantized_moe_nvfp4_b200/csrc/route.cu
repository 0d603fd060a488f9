// route.cu -- token permutation: group the (token, slot) pairs of one MoE layer by expert.
//
// Page "GLM-5-NVFP4-MTP", "Model Description": every token is routed to 8 of 256 experts.
// The expert MLPs run expert by expert, so the T*K pairs are counted per expert (histogram),
// offset by an exclusive prefix sum, and scattered stably (ascending t*K+k within an
// expert) so the result does not depend on thread timing.
//
// One CTA of 1024 threads does the whole job: T*K is at most a few tens of thousands, so
// the step is latency-bound and a single CTA avoids a second launch for the global scan.
// Pairs are taken 1024 at a time; inside a chunk each warp ranks equal ids with
// __match_any_sync, and a per-(warp, expert) table turns warp ranks into positions.
#include "moe.cuh"

namespace nvfp4 {

__global__ void __launch_bounds__(1024) route_kernel(RouteArgs a) {
  extern __shared__ int32_t sm[];
  const int E = a.E;
  int32_t *cnt = sm;             // [E]
  int32_t *base = sm + E;        // [E] next free position per expert
  int32_t *wpos = sm + 2 * E;    // [32][E] position of a warp's first pair of an expert
  __shared__ int32_t s_bad;
  __shared__ int32_t s_nact;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t n = a.n_pairs;

  pdl_wait();  // the ids may come from the previous kernel in the stream
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  if (tid == 0) s_bad = 0;
  __syncthreads();

  // 1. histogram
  int bad = 0;
  for (int64_t p = tid; p < n; p += blockDim.x) {
    const int id = a.map.local(a.ids[p]);
    if (id >= 0)
      atomicAdd(&cnt[id], 1);
    else if (id == kIdBad)
      bad = 1;
  }
  if (bad) atomicOr(&s_bad, 1);
  __syncthreads();

  // 2. exclusive scan of the counts (warp 0, each lane a contiguous run of experts)
  if (warp == 0) {
    const int per = (E + 31) / 32;
    const int e0 = lane * per, e1 = min(E, e0 + per);
    int run = 0, act = 0;
    for (int e = e0; e < e1; ++e) {
      run += cnt[e];
      act += cnt[e] > 0;
    }
    int incl = run, iact = act;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      int w = __shfl_up_sync(0xFFFFFFFFu, iact, o);
      if (lane >= o) {
        incl += v;
        iact += w;
      }
    }
    int pos = incl - run, apos = iact - act;
    for (int e = e0; e < e1; ++e) {
      const int c = cnt[e];
      base[e] = pos;
      if (a.counts) a.counts[e] = c;
      if (a.offsets) a.offsets[e] = pos;
      if (c > 0) {
        if (a.active) a.active[apos] = e;
        ++apos;
      }
      pos += c;
    }
    if (lane == 31) {
      if (a.offsets) a.offsets[E] = pos;
      s_nact = apos;
      if (a.n_active) *a.n_active = apos;
    }
  }
  __syncthreads();

  // 2b. n-tile prefix over the active experts (for the grouped GEMM's tile scheduler)
  if (a.tile_prefix && warp == 0) {
    const int nact = s_nact;
    int run = 0;
    for (int i0 = 0; i0 < nact; i0 += 32) {
      const int i = i0 + lane;
      int nt = 0;
      if (i < nact) nt = (cnt[a.active[i]] + a.tile_n - 1) / a.tile_n;
      int incl = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      if (i < nact) a.tile_prefix[i] = run + incl - nt;
      run += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) a.tile_prefix[nact] = run;
  }

  // 3. stable scatter, 1024 pairs per chunk
  for (int64_t c0 = 0; c0 < n; c0 += blockDim.x) {
    for (int i = tid; i < 32 * E; i += blockDim.x) wpos[i] = 0;
    __syncthreads();
    const int64_t p = c0 + tid;
    const int id = p < n ? a.map.local(a.ids[p]) : kIdBad;
    const bool valid = id >= 0;
    // invalid pairs get a key no valid id can match, unique per lane
    const unsigned key = valid ? (unsigned)id : 0x80000000u | (unsigned)lane;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (valid && rank == 0) wpos[warp * E + id] = __popc(peers);
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
      int run = base[e];
      for (int w = 0; w < 32; ++w) {
        const int c = wpos[w * E + e];
        wpos[w * E + e] = run;
        run += c;
      }
      base[e] = run;
    }
    __syncthreads();
    if (p < n) {
      if (valid) {
        const int pos = wpos[warp * E + id] + rank;
        a.perm[pos] = (int32_t)p;
        if (a.inv) a.inv[p] = pos;
      } else if (a.inv) {
        a.inv[p] = -1;
      }
    }
    __syncthreads();
  }
  // the route step starts a forward call: it (re)writes the whole flag
  if (tid == 0 && a.flag) *a.flag = s_bad ? kFlagBadId : 0;
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ many pairs: three kernels
// Above kRouteChunk pairs the step runs over many CTAs: each chunk of kRouteChunk pairs is
// counted by its own CTA (route_count_kernel), one CTA scans the counts over chunks and
// experts (route_scan_kernel: the tables, and each chunk's first position per expert), and
// each chunk's CTA then scatters its pairs from those positions in the same 1024-pair steps
// as route_kernel (route_scatter_kernel).  The result is the same, position for position.
// blk holds nb * E chunk counts (then positions), followed by nb bad-id bits.

__global__ void __launch_bounds__(1024) route_count_kernel(RouteArgs a, int32_t *blk) {
  extern __shared__ int32_t cnt[];   // [E]
  __shared__ int32_t s_bad;
  const int E = a.E, tid = threadIdx.x;
  const int64_t n = a.n_pairs, p0 = (int64_t)blockIdx.x * kRouteChunk;
  const int64_t p1 = min(n, p0 + kRouteChunk);
  pdl_wait();   // the ids may come from the previous kernel in the stream
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  int bad = 0;
  for (int64_t p = p0 + tid; p < p1; p += blockDim.x) {
    const int id = a.map.local(a.ids[p]);
    if (id >= 0)
      atomicAdd(&cnt[id], 1);
    else if (id == kIdBad)
      bad = 1;
  }
  if (bad) atomicOr(&s_bad, 1);
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) blk[(int64_t)blockIdx.x * E + e] = cnt[e];
  if (tid == 0) blk[(int64_t)gridDim.x * E + blockIdx.x] = s_bad;
  pdl_launch_dependents();
}

__global__ void __launch_bounds__(1024) route_scan_kernel(RouteArgs a, int32_t *blk, int nb) {
  extern __shared__ int32_t sm[];
  const int E = a.E;
  int32_t *cnt = sm;        // [E] pairs per expert
  int32_t *off = sm + E;    // [E] first position per expert
  __shared__ int32_t s_bad;
  __shared__ int32_t s_nact;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();   // the chunk counts
  for (int e = tid; e < E; e += blockDim.x) {
    int c = 0;
    for (int b = 0; b < nb; ++b) c += __ldcg(blk + (int64_t)b * E + e);
    cnt[e] = c;
  }
  if (tid == 0) {
    int bad = 0;
    for (int b = 0; b < nb; ++b) bad |= __ldcg(blk + (int64_t)nb * E + b);
    s_bad = bad;
  }
  __syncthreads();
  if (warp == 0) {   // exclusive scan of the counts, each lane a contiguous run of experts
    const int per = (E + 31) / 32;
    const int e0 = lane * per, e1 = min(E, e0 + per);
    int run = 0, act = 0;
    for (int e = e0; e < e1; ++e) {
      run += cnt[e];
      act += cnt[e] > 0;
    }
    int incl = run, iact = act;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      const int w = __shfl_up_sync(0xFFFFFFFFu, iact, o);
      if (lane >= o) {
        incl += v;
        iact += w;
      }
    }
    int pos = incl - run, apos = iact - act;
    for (int e = e0; e < e1; ++e) {
      const int c = cnt[e];
      off[e] = pos;
      if (a.counts) a.counts[e] = c;
      if (a.offsets) a.offsets[e] = pos;
      if (c > 0) {
        if (a.active) a.active[apos] = e;
        ++apos;
      }
      pos += c;
    }
    if (lane == 31) {
      if (a.offsets) a.offsets[E] = pos;
      s_nact = apos;
      if (a.n_active) *a.n_active = apos;
    }
  }
  __syncthreads();
  if (a.tile_prefix && warp == 0) {   // n-tile prefix over the active experts
    const int nact = s_nact;
    int run = 0;
    for (int i0 = 0; i0 < nact; i0 += 32) {
      const int i = i0 + lane;
      int nt = 0;
      if (i < nact) nt = (cnt[a.active[i]] + a.tile_n - 1) / a.tile_n;
      int incl = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      if (i < nact) a.tile_prefix[i] = run + incl - nt;
      run += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) a.tile_prefix[nact] = run;
  }
  // each chunk's first position per expert: the expert's offset plus the earlier chunks
  for (int e = tid; e < E; e += blockDim.x) {
    int run = off[e];
    for (int b = 0; b < nb; ++b) {
      const int c = __ldcg(blk + (int64_t)b * E + e);
      blk[(int64_t)b * E + e] = run;
      run += c;
    }
  }
  // the route step starts a forward call: it (re)writes the whole flag
  if (tid == 0 && a.flag) *a.flag = s_bad ? kFlagBadId : 0;
  pdl_launch_dependents();
}

__global__ void __launch_bounds__(1024) route_scatter_kernel(RouteArgs a, const int32_t *blk) {
  extern __shared__ int32_t sm[];
  const int E = a.E;
  int32_t *base = sm;        // [E] next free position per expert
  int32_t *wpos = sm + E;    // [32][E] position of a warp's first pair of an expert
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t n = a.n_pairs, p0 = (int64_t)blockIdx.x * kRouteChunk;
  const int64_t p1 = min(n, p0 + kRouteChunk);
  pdl_wait();   // the chunk positions
  for (int e = tid; e < E; e += blockDim.x) base[e] = __ldcg(blk + (int64_t)blockIdx.x * E + e);
  __syncthreads();
  for (int64_t c0 = p0; c0 < p1; c0 += blockDim.x) {
    for (int i = tid; i < 32 * E; i += blockDim.x) wpos[i] = 0;
    __syncthreads();
    const int64_t p = c0 + tid;
    const int id = p < p1 ? a.map.local(a.ids[p]) : kIdBad;
    const bool valid = id >= 0;
    const unsigned key = valid ? (unsigned)id : 0x80000000u | (unsigned)lane;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (valid && rank == 0) wpos[warp * E + id] = __popc(peers);
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
      int run = base[e];
      for (int w = 0; w < 32; ++w) {
        const int c = wpos[w * E + e];
        wpos[w * E + e] = run;
        run += c;
      }
      base[e] = run;
    }
    __syncthreads();
    if (p < p1) {
      if (valid) {
        const int pos = wpos[warp * E + id] + rank;
        a.perm[pos] = (int32_t)p;
        if (a.inv) a.inv[p] = pos;
      } else if (a.inv) {
        a.inv[p] = -1;
      }
    }
    __syncthreads();
  }
  pdl_launch_dependents();
}

size_t route_smem_bytes(int E) { return sizeof(int32_t) * (size_t)E * 34; }

int64_t route_scratch_ints(int64_t n_pairs, int E) {
  const int64_t nb = ceil_div(n_pairs, kRouteChunk);
  return nb * E + nb;
}

static int raise_smem(const void *fn, size_t smem) {
  if (smem <= 48 * 1024) return NVFP4_OK;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  return NVFP4_OK;
}

int launch_route_multi(const RouteArgs &a, int32_t *blk, cudaStream_t stream) {
  const int nb = (int)ceil_div(a.n_pairs, kRouteChunk);
  const size_t smem_count = sizeof(int32_t) * (size_t)a.E;
  const size_t smem_scan = 2 * sizeof(int32_t) * (size_t)a.E;
  const size_t smem_scatter = sizeof(int32_t) * (size_t)a.E * 33;
  if (int s = raise_smem(reinterpret_cast<const void *>(route_scatter_kernel), smem_scatter))
    return s;
  if (int s = launch_pdl(route_count_kernel, dim3(nb), dim3(1024), smem_count, stream, a, blk))
    return s;
  if (int s = launch_pdl(route_scan_kernel, dim3(1), dim3(1024), smem_scan, stream, a, blk, nb))
    return s;
  return launch_pdl(route_scatter_kernel, dim3(nb), dim3(1024), smem_scatter, stream, a,
                    (const int32_t *)blk);
}

int launch_route(const RouteArgs &a, cudaStream_t stream, bool pdl, int32_t *scratch) {
  if (scratch && a.n_pairs > kRouteChunk) return launch_route_multi(a, scratch, stream);
  const size_t smem = route_smem_bytes(a.E);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
      set_last_cuda_error(e);
      return NVFP4_ECUDA;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(1024);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, route_kernel, a);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  return NVFP4_OK;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" int moe_nvfp4_route(const int32_t *topk_ids, int64_t T, int64_t K, int64_t E,
                               int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv,
                               int32_t *error_flag, cudaStream_t stream) {
  if (!topk_ids || !counts || !offsets || !perm || !inv || T <= 0 || K <= 0 || E <= 0)
    return NVFP4_EINVAL;
  if (E > kMaxExperts || K > 16 || T * K >= (int64_t(1) << 31)) return NVFP4_ESHAPE;
  RouteArgs a = {};
  a.ids = topk_ids;
  a.n_pairs = T * K;
  a.E = (int)E;
  a.map = whole_layer(E);
  a.counts = counts;
  a.offsets = offsets;
  a.perm = perm;
  a.inv = inv;
  a.flag = error_flag;
  return launch_route(a, stream, false);
}
