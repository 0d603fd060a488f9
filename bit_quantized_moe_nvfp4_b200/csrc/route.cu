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
#include "route.cuh"

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

size_t route_smem_bytes(int E) { return sizeof(int32_t) * (size_t)E * 34; }

int launch_route(const RouteArgs &a, cudaStream_t stream, bool pdl) {
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
