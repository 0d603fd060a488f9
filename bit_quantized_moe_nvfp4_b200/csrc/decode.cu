// decode.cu -- memory-bound GEMV path of the NVFP4 MoE layer (few tokens per expert).
//
// Page "GLM-5-NVFP4-MTP", "Model Description": the experts are NVFP4 (4-bit values with one
// FP8 scale per 16 elements), 8 of 256 active per token.  With few tokens per expert the
// layer is a stream of packed expert bytes, so two kernels read every needed weight byte
// exactly once:
//
//   gemv_gateup: a_j = g_gu * (W_gu[j] . x) for the gate row j and the up row I+j of each
//                active expert, then h_j = bf16(silu(gate) * up)        (SwiGLU fused)
//   gemv_down:   y_k = g_dn * (W_dn . h_k) for every routed pair, then the top-k weighted
//                combine out[t] = bf16(sum_k w[t,k] y_k) in ascending k    (combine fused)
//
// Each CTA routes the tokens itself (histogram of the ids, exclusive scan, stable ranks) so
// no separate routing launch is needed.  One producer warp streams expert rows into a
// shared-memory ring with 1-D bulk copies (cp.async.bulk, completion counted on mbarriers),
// a few large copies per stage: the number of copies, more than their bytes, sets the pace.
// With one token, the gate/up CTAs claim their row chunks from a counter in the workspace
// (the last one resets it) and the down CTAs each own a slice of output rows for all
// experts; with several tokens each CTA takes a contiguous range of tiles.  The compute
// warps hold the activations as f16 with an exact per-token power-of-two scale; they decode
// E2M1 pairs and E4M3 scales with the hardware converts and accumulate either with
// mixed-precision fma.rn.f32.f16 (one token) or with mma.sync on f16 operands (several
// tokens); f16 x f16 products are exact and sums fp32.  Partial sums are combined across
// lanes by shuffles and across warps through shared memory.
//
// Activation scaling: x_t is multiplied by 2^p_t with p_t = 14 - floor(log2 max|x_t|) and
// rounded to f16.  bf16 has 8 significant bits and f16 11, so this is exact for every
// element above 2^-31 * max|x_t| (smaller ones lose bits below f16's subnormal grid); the
// dot products are rescaled by 2^-p_t in fp32.

#include "moe.cuh"
#include "pipeline.cuh"

namespace nvfp4 {

namespace {

// Stage geometry (compile-time tunables; the defaults are the measured best on B200).
#ifndef NVFP4_GEMV_STAGES
#define NVFP4_GEMV_STAGES 2
#endif
#ifndef NVFP4_GEMV_PAIRS
#define NVFP4_GEMV_PAIRS 8
#endif
#ifndef NVFP4_GEMV_DOWN_ROWS
#define NVFP4_GEMV_DOWN_ROWS 32
#endif
#ifndef NVFP4_GEMV_CTAS_PER_SM
#define NVFP4_GEMV_CTAS_PER_SM 2
#endif
#ifndef NVFP4_GEMV_DOWN_STAGES
#define NVFP4_GEMV_DOWN_STAGES NVFP4_GEMV_STAGES
#endif
#ifndef NVFP4_GEMV_DOWN_SPLIT
#define NVFP4_GEMV_DOWN_SPLIT 1
#endif
#ifndef NVFP4_GEMV_DOWN_WARPS
#define NVFP4_GEMV_DOWN_WARPS 4
#endif
#ifndef NVFP4_GEMV_DOWN_CTAS_PER_SM
#define NVFP4_GEMV_DOWN_CTAS_PER_SM 2
#endif
constexpr int kStages = NVFP4_GEMV_STAGES;       // shared-memory ring depth
constexpr int kPairs = NVFP4_GEMV_PAIRS;         // gate/up row pairs per stage
constexpr int kDownRows = NVFP4_GEMV_DOWN_ROWS;  // rows per stage (down kernel)
constexpr int kDownStages = NVFP4_GEMV_DOWN_STAGES;
constexpr int kDownWarps = NVFP4_GEMV_DOWN_WARPS;   // compute warps (down kernel)
constexpr int kDownSplit = NVFP4_GEMV_DOWN_SPLIT;   // stages per expert (down kernel)
constexpr int kMaxConsumerWarps = 6;
constexpr int64_t kGemvMaxPairs = 1024;  // T*K handled by the GEMV path

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// ------------------------------------------------------------------ small helpers
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Sum each of M per-lane values over the warp (M a power of two <= 32) by recursive
// halving: afterwards lane l holds the total of value index (l >> (5 - log2 M)).
template <int M>
__device__ __forceinline__ float warp_reduce_many(float (&v)[M], int lane) {
#pragma unroll
  for (int width = M; width > 1; width >>= 1) {
    const int d = (16 * width) / M;
    const bool upper = (lane & d) != 0;
#pragma unroll
    for (int i = 0; i < width / 2; ++i) {
      const float send = upper ? v[i] : v[i + width / 2];
      const float keep = upper ? v[i + width / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, d);
    }
  }
  float r = v[0];
#pragma unroll
  for (int d = 16 / M; d >= 1; d >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, d);
  return r;
}

template <int M>
struct Log2 {
  static constexpr int value = (M <= 1) ? 0 : 1 + Log2<M / 2>::value;
};
template <>
struct Log2<1> {
  static constexpr int value = 0;
};

// v[i] for a runtime i < N without dynamic register indexing.
template <int N, typename V>
__device__ __forceinline__ V pick(const V (&v)[N], int i) {
  V r = v[0];
#pragma unroll
  for (int k = 1; k < N; ++k)
    if (i == k) r = v[k];
  return r;
}


// 2 x f32 -> f16x2 (round to nearest even)
__device__ __forceinline__ uint32_t f16x2_rn(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// acc += lo(q) * lo(x) and acc2 += hi(q) * hi(x), f16 operands, fp32 accumulate.
__device__ __forceinline__ void fma_f16x2_f32(uint32_t q, uint32_t x, float &acc, float &acc2) {
  asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %2;\n\tmov.b32 {b0, b1}, %3;\n\t"
      "fma.rn.f32.f16 %0, a0, b0, %0;\n\tfma.rn.f32.f16 %1, a1, b1, %1;\n\t}"
      : "+f"(acc), "+f"(acc2)
      : "r"(q), "r"(x));
}

// Dot of 16 E2M1 codes (two words) with 16 f16 activations (8 f16x2 registers), fp32.
__device__ __forceinline__ float dot16(uint32_t w0, uint32_t w1, const uint32_t *xh) {
  uint32_t q[8];
  e2m1x8_to_f16x2x4(w0, *reinterpret_cast<uint32_t(*)[4]>(&q[0]));
  e2m1x8_to_f16x2x4(w1, *reinterpret_cast<uint32_t(*)[4]>(&q[4]));
  float a = 0.f, b = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) fma_f16x2_f32(q[i], xh[i], a, b);
  return a + b;
}


// ------------------------------------------------------------------ in-CTA routing
// Shared-memory routing tables of one CTA.
struct CtaRoute {
  int *ids;      // [n]  expert id of pair p (copy of topk_ids)
  int *act_e;    // [min(E, n)]  active experts, ascending
  int *act_off;  // [min(E, n) + 1]  first slot of each active expert
  int *n_act;    // [1]
};

// All threads of the CTA: copy the ids as local experts (kIdForeign / kIdBad for pairs
// this device does not serve), count pairs per local expert (hist[E] is scratch), and
// list the active experts with the exclusive prefix of their counts.  hist[e] ends up as
// the active index of expert e (-1 if none).  Returns true if some id is out of range.
__device__ bool cta_route(const int32_t *g_ids, int n, int E, ExpertMap map, CtaRoute r,
                          int *hist) {
  __shared__ int s_bad;
  const int tid = threadIdx.x, nth = blockDim.x, lane = tid & 31;
  if (tid == 0) s_bad = 0;
  for (int e = tid; e < E; e += nth) hist[e] = 0;
  // ids are read past L1: they may have been written by the kernel this one follows
  for (int p = tid; p < n; p += nth) r.ids[p] = map.local(__ldcg(g_ids + p));
  __syncthreads();
  bool bad = false;
  for (int p = tid; p < n; p += nth) {
    const int v = r.ids[p];
    if (v >= 0)
      atomicAdd(&hist[v], 1);
    else if (v == kIdBad)
      bad = true;
  }
  if (bad) s_bad = 1;
  __syncthreads();
  if (tid < 32) {
    const int per = (E + 31) / 32;
    const int e0 = lane * per, e1 = min(E, e0 + per);
    int run = 0, act = 0;
    for (int e = e0; e < e1; ++e) {
      run += hist[e];
      act += hist[e] > 0;
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
      const int c = hist[e];
      if (c > 0) {
        r.act_e[apos] = e;
        r.act_off[apos] = pos;
        hist[e] = apos;
        ++apos;
      } else {
        hist[e] = -1;
      }
      pos += c;
    }
    if (lane == 31) {
      r.act_off[apos] = pos;
      *r.n_act = apos;
    }
  }
  __syncthreads();
  return s_bad != 0;
}

// The pairs p (ascending) routed to expert e with rank in [first, first + NT): lane i < NT
// of the calling warp receives the i-th one (-1 past the end).
template <int NT>
__device__ int pairs_of_expert(const int *ids, int n, int e, int first, int lane) {
  int seen = 0, mine = -1;
  for (int base = 0; base < n && seen < first + NT; base += 32) {
    const int p = base + lane;
    const bool m = p < n && ids[p] == e;
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, m);
    const int rank = seen + __popc(bal & ((1u << lane) - 1u));
    // hand pair p to lane (rank - first)
    const int want = lane + first;   // the rank lane `lane` is looking for
#pragma unroll 1
    for (unsigned b = bal; b; b &= b - 1) {
      const int src = __ffs(b) - 1;
      const int rk = __shfl_sync(0xFFFFFFFFu, rank, src);
      if (rk == want) mine = base + src;
    }
    seen += __popc(bal);
  }
  return lane < NT ? mine : -1;
}

// Slot (row of h) of every pair: slot = first slot of its expert + stable rank; -1 for a
// pair this device does not serve.  ids are local (cta_route).  One warp; run[] is scratch
// of n_act ints.
__device__ void warp_slots(const int *ids, int n, const int *act_index, const int *act_off,
                           int n_act, int *run, int *slot, int lane) {
  for (int a = lane; a < n_act; a += 32) run[a] = act_off[a];
  __syncwarp();
  for (int base = 0; base < n; base += 32) {
    const int p = base + lane;
    const int v = p < n ? ids[p] : kIdBad;
    const bool valid = v >= 0;
    const unsigned key = valid ? (unsigned)v : 0x80000000u | (unsigned)lane;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int ai = valid ? act_index[v] : -1;
    const int s = valid ? run[ai] + rank : -1;
    __syncwarp();
    if (valid && rank == 0) run[ai] += __popc(peers);
    __syncwarp();
    if (p < n) slot[p] = s;
  }
}

// Load one activation slice (32 bf16 at src) for a lane, return its max |x| (fp32).
__device__ __forceinline__ float load_bf16x32(const __nv_bfloat16 *src, uint4 (&v)[4]) {
  const uint4 *p = reinterpret_cast<const uint4 *>(src);
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[i] = __ldcg(p + i);
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[k])), fabsf(bf16_hi(w[k]))));
  }
  return m;
}

// 32 bf16 -> 16 f16x2 after scaling by s (exact power of two)
__device__ __forceinline__ void to_f16x32(const uint4 (&v)[4], float s, uint32_t *xh) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) xh[4 * i + k] = f16x2_rn(bf16_lo(w[k]) * s, bf16_hi(w[k]) * s);
  }
}

// Shared memory carve-up common to both kernels (offsets in bytes from the dynamic base).
// Barriers: full[S] / empty[S] for the stage ring, rfull[R] / rfree[R] for the ring of
// reduction slots that carries partial sums from the consumer warps to the finalizer warp.
constexpr int kRedSlots = 4;

struct Smem {
  uint32_t bars, stages, red, smax, ids, act_e, act_off, misc, slot, run, hist, yk, hpre, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Floats per reduction slot: CW * red_vals partial sums + 2 * 4 per-token extras.
__host__ __device__ inline int red_slot_floats(int cw, int red_vals) { return cw * red_vals + 8; }

__host__ __device__ inline Smem smem_layout(int S, uint32_t stage_bytes, int cw, int red_vals,
                                            int n, int E, int yk_floats, uint32_t hpre_bytes = 0) {
  Smem s;
  uint32_t o = 0;
  s.bars = o;
  o += 8 * (2 * S + 2 * kRedSlots);
  o = align_up(o, 128);
  s.stages = o;
  o += stage_bytes * S;
  s.red = o;
  o += 4 * kRedSlots * red_slot_floats(cw, red_vals);
  s.smax = o;
  o += 4 * (cw * 8 + 8);
  s.ids = o;
  o += 4 * n;
  const int na = min(E, n);
  s.act_e = o;
  o += 4 * na;
  s.act_off = o;
  o += 4 * (na + 1);
  s.misc = o;
  o += 16;
  s.slot = o;
  o += 4 * n;
  s.run = o;
  o += 4 * na;
  s.hist = o;
  o += 4 * E;
  o = align_up(o, 16);
  s.yk = o;
  o += 4 * yk_floats;
  o = align_up(o, 16);
  s.hpre = o;
  o += hpre_bytes;
  s.total = align_up(o, 128);
  return s;
}

// Wait on an mbarrier phase with the whole warp agreeing on the outcome.  Once any wait of
// the CTA has given up (abort set), later waits are skipped and report failure, so every
// role still runs its loops to the end (arrivals included) without blocking.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int *abort,
                                          int32_t *flag) {
  bool ok = false;
  if (!*(volatile int *)abort) ok = mbar_wait(bar, parity);
  ok = __all_sync(0xFFFFFFFFu, ok);
  if (!ok && !*(volatile int *)abort && (threadIdx.x & 31) == 0) {
    *(volatile int *)abort = 1;
    report_timeout(flag);
  }
  return ok;
}

// ================================================================== gate/up + SwiGLU
// blockDim = 32 * (CW + 2): warp 0 produces (bulk copies), warps 1..CW compute, warp CW+1
// finalizes.  Each computing lane owns 32 consecutive elements (16 packed bytes, 2 block
// scales) of every row; a stage holds P gate rows and the P matching up rows of one expert.
template <int NT, int P, int S>
__global__ void __launch_bounds__(32 * (kMaxConsumerWarps + 2), NT == 1 ? 2 : 1)
    gemv_gateup_kernel(MoeArgs a, uint32_t stage_bytes) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_abort;
  const int CW = blockDim.x / 32 - 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t H = a.H, I = a.I, K = a.K;
  const int n = (int)(a.T * K);
  const int E = (int)a.E;
  constexpr int RV = 2 * P * NT;   // values reduced per stage per lane
  const int RS = red_slot_floats(CW, RV);
  const Smem L = smem_layout(S, stage_bytes, CW, RV, n, E, 0);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *empty = full + S;
  uint64_t *rfull = empty + S;
  uint64_t *rfree = rfull + kRedSlots;
  unsigned char *stage_base = smem + L.stages;
  float *red = reinterpret_cast<float *>(smem + L.red);
  float *smax = reinterpret_cast<float *>(smem + L.smax);
  CtaRoute R{reinterpret_cast<int *>(smem + L.ids), reinterpret_cast<int *>(smem + L.act_e),
             reinterpret_cast<int *>(smem + L.act_off), reinterpret_cast<int *>(smem + L.misc)};
  int *hist = reinterpret_cast<int *>(smem + L.hist);

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    for (int s = 0; s < kRedSlots; ++s) {
      mbar_init(&rfull[s], CW);
      mbar_init(&rfree[s], 1);
    }
    mbar_init_fence();
  }
  pdl_wait();  // x and the ids come from earlier kernels
  // One token: the compute lanes issue their activation loads first, so they are not
  // queued behind the weight stream that starts once the routing is known.
  const int chunk = (warp - 1) * 32 + lane;      // 32-element chunk owned by a compute lane
  const bool owns = warp >= 1 && warp <= CW && chunk < (int)(H / 32);
  uint4 xv[4];
  if (NT == 1 && owns) {
    const uint4 *xp = reinterpret_cast<const uint4 *>(a.x + chunk * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i) xv[i] = __ldcg(xp + i);
  }
  const bool bad = cta_route(a.ids, n, E, a.map, R, hist);
  if (blockIdx.x == 0 && threadIdx.x == 0 && a.flag) *a.flag = bad ? kFlagBadId : 0;
  pdl_launch_dependents();  // the down kernel may start routing and prefetching

  const int n_act = *R.n_act;
  // Work is handed out dynamically: chunk c is pair rows [j, j + P) of active expert c / cpe
  // (j = (c % cpe) * P), claimed by the producers from the counter work[0], so CTAs that got
  // their first stage late do less of it.  A producer holds at most one claimed chunk that
  // it has not issued yet, and stops at its first claim past the end; the last producer to
  // stop resets the counters.
  const int cpe = (int)ceil_div(I, P);
  const int total = n_act * cpe;
  const uint32_t rowb = (uint32_t)(H / 2), sclb = (uint32_t)(H / 16);
  const uint32_t span_stride = span_bytes(P * sclb);
  __shared__ int s_unit[S], s_np[S];   // per stage: first unit (ai * I + j, -1 = no more), rows

  if (warp == 0) {
    // ------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      int next = atomicAdd(a.work, 1);   // claimed one chunk ahead: the atomic's round trip
      for (;; ++s) {                     // overlaps the wait for a free stage
        const int idx = s % S;
        if (s >= S && (*(volatile int *)&s_abort || !mbar_wait(&empty[idx], ((s / S) - 1) & 1))) {
          if (!*(volatile int *)&s_abort) report_timeout(a.flag);
          *(volatile int *)&s_abort = 1;
          break;
        }
        const int c = next;
        if (c < total) next = atomicAdd(a.work, 1);
        if (c >= total) {   // tell the consumers to stop (a plain arrive completes the phase)
          s_unit[idx] = -1;
          mbar_arrive(&full[idx]);
          ++s;
          break;
        }
        const int ai = c / cpe;
        const int64_t j = (int64_t)(c % cpe) * P;
        const int np = (int)min64(P, I - j);
        const int e = R.act_e[ai];
        s_unit[idx] = (int)(ai * I + j);
        s_np[idx] = np;
        unsigned char *st = stage_base + (size_t)idx * stage_bytes;
        const int64_t rg = (int64_t)e * 2 * I + j;   // first gate row
        const int64_t ru = rg + I;                   // first up row
        const uint8_t *sblock = a.s_gu + (int64_t)e * 2 * I * sclb;
        const int64_t lg = j * sclb, lu = (I + j) * sclb;   // offsets inside the block
        const uint32_t span_g = (uint32_t)(((lg + np * sclb + 15) & ~15ll) - (lg & ~15ll));
        const uint32_t span_u = (uint32_t)(((lu + np * sclb + 15) & ~15ll) - (lu & ~15ll));
        mbar_arrive_expect_tx(&full[idx], 2u * np * rowb + span_g + span_u);
        bulk_g2s(st, a.w_gu + rg * rowb, np * rowb, &full[idx]);
        bulk_g2s(st + P * rowb, a.w_gu + ru * rowb, np * rowb, &full[idx]);
        unsigned char *sc = st + 2 * P * rowb;
        bulk_g2s_span(sc, sblock, lg, np * sclb, &full[idx]);
        bulk_g2s_span(sc + span_stride, sblock, lu, np * sclb, &full[idx]);
      }
      // this CTA claims nothing more: the last CTA to get here resets the counters
      __threadfence();
      if (atomicAdd(a.work + 1, 1) == (int)gridDim.x - 1) {
        atomicExch(a.work, 0);
        atomicExch(a.work + 1, 0);
      }
      // do not leave while copies into this CTA's shared memory may still be in flight
      const int issued = s;
      for (int t = max(0, issued - S); t < issued; ++t)
        if (!mbar_wait(&full[t % S], (t / S) & 1)) report_timeout(a.flag);
    }
    return;
  }

  if (warp == CW + 1) {
    // ------------------------------------------------ finalizer
    // Each reduction slot carries its stage's first unit, rows and token group; a unit of -1
    // marks the end.
    int cur_a = -1, slot0 = 0, cnt = 0;
    float g = 0.f;
    for (int it = 0;; ++it) {
      const int sl = it % kRedSlots;
      if (!warp_wait(&rfull[sl], (it / kRedSlots) & 1, &s_abort, a.flag)) break;
      const float *rb = red + (size_t)sl * RS;
      const int u = __float_as_int(rb[CW * RV + 4]);
      if (u < 0) break;
      const int np = __float_as_int(rb[CW * RV + 5]);
      const int grp = __float_as_int(rb[CW * RV + 6]);
      const int ai = u / (int)I;
      const int64_t j = u % (int)I;
      if (ai != cur_a) {
        cur_a = ai;
        slot0 = R.act_off[ai];
        cnt = R.act_off[ai + 1] - slot0;
        g = __ldg(a.g_gu + R.act_e[ai]);
      }
      const int nt = min(NT, cnt - grp * NT);
      if (lane < np * nt) {
        const int pp = lane / nt, i = lane % nt;
        float gs = 0.f, us = 0.f;
        for (int w = 0; w < CW; ++w) {
          gs += rb[w * RV + pp * NT + i];
          us += rb[w * RV + (P + pp) * NT + i];
        }
        const float ps = rb[CW * RV + i];
        const float gate = gs * g * ps;
        const float up = us * g * ps;
        const int slot = slot0 + grp * NT + i;
        a.h[(int64_t)slot * I + j + pp] = __float2bfloat16_rn(silu_f32(gate) * up);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rfree[sl]);
    }
    return;
  }

  // ------------------------------------------------ compute warps
  const int cw = warp - 1;                       // compute warp index
  const int nthreads_c = CW * 32;
  uint32_t xh[NT][16];
  float pscale[NT];                              // 2^-p per token of the current group
  int loaded_tok[NT];                            // tokens whose activations are in xh
#pragma unroll
  for (int i = 0; i < NT; ++i) loaded_tok[i] = -1;
  int cur_a = -1, ngroups = 0, cnt = 0;
  int s = 0, it = 0;
  if (NT == 1) {
    // One token: every pair is token 0, whose activations were loaded above; they are
    // scaled to f16 before the first stage arrives.
    float mx = 0.f;
    if (owns) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t w4[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mx = fmaxf(mx, fmaxf(fabsf(bf16_lo(w4[k])), fabsf(bf16_hi(w4[k]))));
      }
    }
    const float m = warp_max(mx);
    if (lane == 0) smax[cw * 4] = m;
    named_sync(1, nthreads_c);
    float mm = 0.f;
    for (int w = 0; w < CW; ++w) mm = fmaxf(mm, smax[w * 4]);
    const int p = prescale_exponent(mm);
    pscale[0] = exp2i(-p);
    if (owns) to_f16x32(xv, exp2i(p), xh[0]);
    loaded_tok[0] = 0;
    named_sync(1, nthreads_c);   // smax is rewritten by any later load
  }
  for (;; ++s) {
    const int idx = s % S;
    const bool have = warp_wait(&full[idx], (s / S) & 1, &s_abort, a.flag);
    const int u = have ? s_unit[idx] : -1;   // written before the producer's arrive
    if (u < 0) break;                          // no more stages (or a wait gave up)
    const int np = s_np[idx];
    const int ai = u / (int)I;
    const int64_t j = u % (int)I;
    const bool new_expert = ai != cur_a;
    if (new_expert) {
      cur_a = ai;
      cnt = R.act_off[ai + 1] - R.act_off[ai];
      ngroups = (cnt + NT - 1) / NT;
    }
    const unsigned char *st = stage_base + (size_t)idx * stage_bytes;
    const int64_t offg = j * sclb, offu = (I + j) * sclb;
    const unsigned char *spg = st + 2 * P * rowb + (offg & 15);
    const unsigned char *spu = st + 2 * P * rowb + span_stride + (offu & 15);
    for (int grp = 0; grp < ngroups; ++grp, ++it) {
      const int nt = min(NT, cnt - grp * NT);
      const bool last = grp == ngroups - 1;
      // (re)load the activations of this token group when they are not in registers
      bool reload = false;
      int tok[NT];
      if (ngroups > 1 || new_expert) {
        // the same tokens as the ones in registers (always so for a single token) need no
        // reload; the decision depends only on shared data, so all compute warps agree
        const int pr = pairs_of_expert<NT>(R.ids, n, R.act_e[ai], grp * NT, lane);
#pragma unroll
        for (int i = 0; i < NT; ++i) {
          tok[i] = (int)(__shfl_sync(0xFFFFFFFFu, pr, min(i, nt - 1)) / K);
          reload |= tok[i] != loaded_tok[i];
        }
      }
      if (reload) {
        const __nv_bfloat16 *xr[NT];
#pragma unroll
        for (int i = 0; i < NT; ++i) {
          loaded_tok[i] = tok[i];
          xr[i] = a.x + (int64_t)tok[i] * H + chunk * 32;
        }
        // pass 1: largest magnitude of each token (over all compute warps)
        float m[NT];
#pragma unroll
        for (int i = 0; i < NT; ++i) {
          uint4 v[4];
          m[i] = warp_max(owns ? load_bf16x32(xr[i], v) : 0.f);
        }
        if (lane == 0)
#pragma unroll
          for (int i = 0; i < NT; ++i) smax[cw * 4 + i] = m[i];
        named_sync(1, nthreads_c);
        // pass 2: scale by 2^p and round to f16 (the reload hits L1/L2)
#pragma unroll
        for (int i = 0; i < NT; ++i) {
          float mm = 0.f;
          for (int w = 0; w < CW; ++w) mm = fmaxf(mm, smax[w * 4 + i]);
          const int p = prescale_exponent(mm);
          pscale[i] = exp2i(-p);
          if (owns) {
            uint4 v[4];
            load_bf16x32(xr[i], v);
            to_f16x32(v, exp2i(p), xh[i]);
          }
        }
        named_sync(1, nthreads_c);   // smax is rewritten by the next load
      }
      // partial dot products of the 2*np loaded rows (the others stay zero and are ignored)
      float flat[RV];
#pragma unroll
      for (int v = 0; v < RV; ++v) flat[v] = 0.f;
      if (owns && have) {
#pragma unroll
        for (int r = 0; r < 2 * P; ++r) {
          if (r % P >= np) continue;   // warp-uniform: a short stage skips its stale rows
          const uint4 q = *reinterpret_cast<const uint4 *>(st + (size_t)r * rowb + chunk * 16);
          const unsigned char *sp = (r < P) ? spg : spu;
          const uint32_t sc2 = *reinterpret_cast<const unsigned short *>(
              sp + (size_t)(r % P) * sclb + chunk * 2);
          const uint32_t s16 = e4m3x2_to_f16x2(sc2);
          const float s0 = f16_lo(s16), s1 = f16_hi(s16);
#pragma unroll
          for (int i = 0; i < NT; ++i) {
            const float d0 = dot16(q.x, q.y, &xh[i][0]);
            const float d1 = dot16(q.z, q.w, &xh[i][8]);
            flat[r * NT + i] = fmaf(d1, s1, d0 * s0);
          }
        }
      }
      if (last) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[idx]);   // this warp is done reading the stage
      }
      const float tot = warp_reduce_many<RV>(flat, lane);
      constexpr int SH = 5 - Log2<RV>::value;
      const int sl = it % kRedSlots;
      if (it >= kRedSlots) warp_wait(&rfree[sl], ((it / kRedSlots) - 1) & 1, &s_abort, a.flag);
      float *rb = red + (size_t)sl * RS;
      if ((lane & ((1 << SH) - 1)) == 0) rb[cw * RV + (lane >> SH)] = tot;
      if (cw == 0 && lane < NT) rb[CW * RV + lane] = pick<NT>(pscale, lane);
      if (cw == 0 && lane == 0) {
        rb[CW * RV + 4] = __int_as_float(u);
        rb[CW * RV + 5] = __int_as_float(np);
        rb[CW * RV + 6] = __int_as_float(grp);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rfull[sl]);
    }
  }
  // end marker for the finalizer
  const int sl = it % kRedSlots;
  if (it >= kRedSlots) warp_wait(&rfree[sl], ((it / kRedSlots) - 1) & 1, &s_abort, a.flag);
  if (cw == 0 && lane == 0) red[(size_t)sl * RS + CW * RV + 4] = __int_as_float(-1);
  __syncwarp();
  if (lane == 0) mbar_arrive(&rfull[sl]);
}

// ================================================================== projections on mma.sync
// Both projections of the GEMV path run on the tensor cores with mma.sync.m16n8k16
// (f16 x f16 -> fp32): M = 16 weight rows of one expert, N = 8 token slots, K = 16.
//   MODE 0, gate/up: rows = gate rows j..j+7 and up rows j..j+7; the activations are x;
//           result h[slot, j+r] = bf16( silu(g_gu * gate_r) * g_gu * up_r )  (SwiGLU)
//   MODE 1, down:    rows = output rows r0..r0+31 (two M-tiles); the activations are the h
//           rows of the expert's slots; result y[pair, r0+r] = w[pair] * g_dn * (W_dn h)_r,
//           combined over k afterwards (combine.cu)
// A unit is one such tile; each CTA takes a contiguous range of units in expert order, so an
// expert's activations are loaded once per CTA.  Since a dot product may sum its terms in any order, the K index of the MMA is
// mapped to memory so that each lane decodes only contiguous bytes: lane (g, t) (g = lane/4,
// t = lane%4) owns elements 32t..32t+31 of every 128-element chunk, for weight rows g and
// g+8 (A operand) and for token g (B operand); MMA i of a chunk takes elements
// 32t+4i..32t+4i+3 of each lane.  E2M1 codes become f16 with the hardware convert and are
// multiplied by their E4M3 block scale in f16 (exact: at most 6 significant bits), the
// activations are f16 with the per-token power-of-two scale, and the tensor core sums in
// fp32.  This takes about a third of the instructions of a CUDA-core dot product per byte.
constexpr int kGuWarps = 16;                  // compute warps
constexpr int kGuFinal = 2;                   // finaliser warps (one per other reduction slot)
constexpr int kGuMaxChunks = 3;               // 128-element chunks per warp: H <= 6144
constexpr int kGuTok = 8;                     // token slots per group (MMA N)
// Tile rows: 16 for gate/up (8 gate + 8 up rows, one MMA M-tile), 32 for down (two M-tiles:
// the down tile is a third of a gate/up tile in bytes, and a tile's fixed cost -- the partial
// sums, the finalisers, the barrier hand-offs -- is then paid once per 32 KB).
__host__ __device__ constexpr int gu_mtiles(int mode) { return mode == 0 ? 1 : 2; }
// Floats per reduction slot: each compute warp's partials (M-tiles x 16 rows x 8 tokens),
// then the 8 tokens' 2^-p and pair indices.
__host__ __device__ constexpr int gu_red_floats(int mode) {
  return kGuWarps * 16 * gu_mtiles(mode) * kGuTok + 2 * kGuTok;
}

__device__ __forceinline__ void mma_16816_f16(float (&d)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0,
                                              uint32_t b1) {
  // not volatile: the MMA has no effect besides its outputs, so the compiler may schedule
  // the decode of the next operands around it
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&a), *reinterpret_cast<const __half2 *>(&b));
  return *reinterpret_cast<uint32_t *>(&r);
}

struct GuSmem {
  uint32_t bars, stages, red, smax, ids, act_e, act_off, misc, hist, wts, total;
};

__host__ __device__ inline GuSmem gu_smem_layout(int S, uint32_t stage_bytes, int n, int E,
                                                 int red_floats) {
  GuSmem s;
  uint32_t o = 0;
  s.bars = o;
  o += 8 * (2 * S + 2 * kRedSlots);
  o = align_up(o, 128);
  s.stages = o;
  o += stage_bytes * S;
  s.red = o;
  o += 4 * kRedSlots * red_floats;
  s.smax = o;
  o += 4 * kGuWarps * kGuTok;
  s.ids = o;
  o += 4 * n;
  const int na = min(E, n);
  s.act_e = o;
  o += 4 * na;
  s.act_off = o;
  o += 4 * (na + 1);
  s.misc = o;
  o += 16;
  s.hist = o;
  o += 4 * E;
  s.wts = o;   // [n] copy of topk_w (down: the finaliser weights each pair's y)
  o += 4 * n;
  s.total = align_up(o, 128);
  return s;
}

// Stage geometry for a reduction length Kd and rows = 16 x M-tiles: the packed rows at a
// stride of Kd/2 bytes (each half of the tile arrives with one bulk copy: per-row copies with
// a bank-spreading pad were slower, the copy count per tile being the limit), then the
// block-scale runs of the two halves.
__host__ __device__ inline uint32_t gu_row_stride(int64_t Kd) { return (uint32_t)(Kd / 2); }
__host__ __device__ inline uint32_t gu_stage_bytes(int64_t Kd, int rows) {
  return rows * gu_row_stride(Kd) + 2 * span_bytes((rows / 2) * (Kd / 16));
}

// blockDim = 32 * (kGuWarps + 1 + kGuFinal): warp 0 produces, warps 1..kGuWarps compute,
// the last kGuFinal warps finalize (finaliser f takes the reduction slots it with
// it % kGuFinal == f, so each slot's barriers have one waiter, in order).  A warp's partial
// sums sit token-major in its slot (token slot tk, tile row r at tk * 16 + r), so the
// finalisers read them without bank conflicts.
// MC: 128-element chunks per compute warp at most (reduction length <= 16 * 128 * MC).
template <int MODE, int S, int MC>
__global__ void __launch_bounds__(32 * (kGuWarps + 1 + kGuFinal), 1)
    gemv_mma_kernel(MoeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_abort;
  constexpr int CW = kGuWarps;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t H = a.H, I = a.I, K = a.K;
  const int64_t Kd = MODE == 0 ? H : I;          // reduction length
  constexpr int MT = gu_mtiles(MODE);            // MMA M-tiles per tile
  constexpr int RT = 16 * MT, HALF = RT / 2;     // rows per tile, rows per bulk copy
  constexpr int RF = gu_red_floats(MODE);        // floats per reduction slot
  const int n = (int)(a.T * K);
  const int E = (int)a.E;
  const uint32_t rstride = gu_row_stride(Kd), stage_bytes = gu_stage_bytes(Kd, RT);
  const GuSmem L = gu_smem_layout(S, stage_bytes, n, E, RF);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *empty = full + S;
  uint64_t *rfull = empty + S;
  uint64_t *rfree = rfull + kRedSlots;
  unsigned char *stage_base = smem + L.stages;
  float *red = reinterpret_cast<float *>(smem + L.red);
  float *smax = reinterpret_cast<float *>(smem + L.smax);
  CtaRoute R{reinterpret_cast<int *>(smem + L.ids), reinterpret_cast<int *>(smem + L.act_e),
             reinterpret_cast<int *>(smem + L.act_off), reinterpret_cast<int *>(smem + L.misc)};
  int *hist = reinterpret_cast<int *>(smem + L.hist);

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    for (int s = 0; s < kRedSlots; ++s) {
      mbar_init(&rfull[s], CW);
      mbar_init(&rfree[s], 1);
    }
    mbar_init_fence();
  }
  if (MODE == 0) pdl_wait();   // x and the ids come from earlier kernels
  // (MODE 1: the ids were complete before the gate/up kernel let this grid start, so the
  // routing and the weight stream start before griddepcontrol.wait)
  const bool bad = cta_route(a.ids, n, E, a.map, R, hist);
  if (MODE == 0 && blockIdx.x == 0 && threadIdx.x == 0 && a.flag) *a.flag = bad ? kFlagBadId : 0;
  float *wts = reinterpret_cast<float *>(smem + L.wts);
  if (MODE == 1) {   // the pair weights, read once here instead of once per tile and output
    for (int p = threadIdx.x; p < n; p += blockDim.x) wts[p] = __ldg(a.w + p);
    __syncthreads();
  }
  pdl_launch_dependents();  // the next kernel may start its prologue

  const int n_act = *R.n_act;
  const int64_t upe = MODE == 0 ? I / 8 : H / RT;   // units (tiles) per expert
  const int64_t units = (int64_t)n_act * upe;
  const int64_t U0 = units * blockIdx.x / gridDim.x, U1 = units * (blockIdx.x + 1) / gridDim.x;
  const uint32_t rowb = (uint32_t)(Kd / 2), sclb = (uint32_t)(Kd / 16);
  const uint32_t scl_off = RT * rstride;
  const uint32_t span_stride = span_bytes(HALF * sclb);

  if (warp == 0) {
    // ------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      for (int64_t u = U0; u < U1; ++u, ++s) {
        const int ai = (int)(u / upe);
        const int e = R.act_e[ai];
        const int idx = s % S;
        if (s >= S && (*(volatile int *)&s_abort || !mbar_wait(&empty[idx], ((s / S) - 1) & 1))) {
          if (!*(volatile int *)&s_abort) report_timeout(a.flag);
          *(volatile int *)&s_abort = 1;
          break;
        }
        unsigned char *st = stage_base + (size_t)idx * stage_bytes;
        // the tile's two halves, as row indices inside the expert's weight block
        const int64_t lr0 = MODE == 0 ? (u % upe) * 8 : (u % upe) * RT;
        const int64_t lr1 = MODE == 0 ? I + lr0 : lr0 + HALF;
        const int64_t rows_pe = MODE == 0 ? 2 * I : H;
        const uint8_t *wblock = (MODE == 0 ? a.w_gu : a.w_dn) + (int64_t)e * rows_pe * rowb;
        const uint8_t *sblock = (MODE == 0 ? a.s_gu : a.s_dn) + (int64_t)e * rows_pe * sclb;
        const int64_t lg = lr0 * sclb, lu = lr1 * sclb;
        const uint32_t span_g = (uint32_t)(((lg + HALF * sclb + 15) & ~15ll) - (lg & ~15ll));
        const uint32_t span_u = (uint32_t)(((lu + HALF * sclb + 15) & ~15ll) - (lu & ~15ll));
        mbar_arrive_expect_tx(&full[idx], (uint32_t)RT * rowb + span_g + span_u);
        bulk_g2s(st, wblock + lr0 * rowb, HALF * rowb, &full[idx]);                 // first half
        bulk_g2s(st + HALF * rstride, wblock + lr1 * rowb, HALF * rowb, &full[idx]);  // second
        bulk_g2s_span(st + scl_off, sblock, lg, HALF * sclb, &full[idx]);
        bulk_g2s_span(st + scl_off + span_stride, sblock, lu, HALF * sclb, &full[idx]);
      }
      const int issued = s;
      for (int t = max(0, issued - S); t < issued; ++t)
        if (!mbar_wait(&full[t % S], (t / S) & 1)) report_timeout(a.flag);
    }
    return;
  }

  if (warp > CW) {
    // ------------------------------------------------ finalizers
    const int fin = warp - CW - 1;
    int it = 0, cur_a = -1, slot0 = 0, cnt = 0;
    float gsc = 0.f;
    for (int64_t u = U0; u < U1; ++u) {
      const int ai = (int)(u / upe);
      const int64_t j = MODE == 0 ? (u % upe) * 8 : (u % upe) * RT;   // first row / pair
      if (ai != cur_a) {
        cur_a = ai;
        slot0 = R.act_off[ai];
        cnt = R.act_off[ai + 1] - slot0;
        gsc = __ldg((MODE == 0 ? a.g_gu : a.g_dn) + R.act_e[ai]);
      }
      for (int grp = 0; grp * kGuTok < cnt; ++grp, ++it) {
        if (it % kGuFinal != fin) continue;
        const int nt = min(kGuTok, cnt - grp * kGuTok);
        const int sl = it % kRedSlots;
        const bool ok = warp_wait(&rfull[sl], (it / kRedSlots) & 1, &s_abort, a.flag);
        const float *rb = red + (size_t)sl * RF;
        if (MODE == 0) {
          for (int q = lane; ok && q < 8 * nt; q += 32) {
            const int tk = q >> 3, r = q & 7;   // token slot of the group, row pair
            float gp[4] = {0.f, 0.f, 0.f, 0.f}, up4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
            for (int w = 0; w < CW; ++w) {     // four chains, summed in a fixed order
              gp[w & 3] += rb[w * 128 * MT + tk * 16 + r];
              up4[w & 3] += rb[w * 128 * MT + tk * 16 + 8 + r];
            }
            const float gs = (gp[0] + gp[1]) + (gp[2] + gp[3]);
            const float us = (up4[0] + up4[1]) + (up4[2] + up4[3]);
            const float ps = rb[CW * 128 * MT + tk];
            const float gate = gs * gsc * ps, up = us * gsc * ps;
            const int slot = slot0 + grp * kGuTok + tk;
            a.h[(int64_t)slot * I + j + r] = __float2bfloat16_rn(silu_f32(gate) * up);
          }
        } else {
          for (int q = lane; ok && q < RT * nt; q += 32) {
            const int tk = q / RT, r = q % RT;  // token slot of the group, tile row
            const int po = (r >> 4) * 128 + tk * 16 + (r & 15);   // M-tile, token, row
            float yp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
            for (int w = 0; w < CW; ++w) yp[w & 3] += rb[w * 128 * MT + po];
            const float ys = (yp[0] + yp[1]) + (yp[2] + yp[3]);
            const float ps = rb[CW * 128 * MT + tk];
            const int pair = __float_as_int(rb[CW * 128 * MT + kGuTok + tk]);
            a.y[(int64_t)pair * H + j + r] = ys * gsc * ps * wts[pair];
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&rfree[sl]);
      }
    }
    return;
  }

  // ------------------------------------------------ compute warps
  if (MODE == 1) pdl_wait();   // h is written by the gate/up kernel
  const int cw = warp - 1;
  const int g = lane >> 2, t = lane & 3;
  const int nchunk = (int)((Kd + 127) / 128);
  const int nthreads_c = CW * 32;
  uint32_t xr[MC][16];     // token g's activations (f16x2), chunk cw + CW*m
  float pscale = 1.f;                // 2^-p of token g
  int loaded_tok = -2;               // activation row that lane group g holds
  int mypair = -1;                   // pair of slot g of the current group
  const __nv_bfloat16 *arow = MODE == 0 ? a.x : a.h;
#pragma unroll
  for (int m = 0; m < MC; ++m)
#pragma unroll
    for (int i = 0; i < 16; ++i) xr[m][i] = 0u;
  int cur_a = -1, ngroups = 0, cnt = 0;
  int s = 0, it = 0;
  for (int64_t u = U0; u < U1; ++u, ++s) {
    const int ai = (int)(u / upe);
    const int64_t lr0 = MODE == 0 ? (u % upe) * 8 : (u % upe) * RT;
    const int64_t lr1 = MODE == 0 ? I + lr0 : lr0 + HALF;
    const int idx = s % S;
    const bool new_expert = ai != cur_a;
    if (new_expert) {
      cur_a = ai;
      cnt = R.act_off[ai + 1] - R.act_off[ai];
      ngroups = (cnt + kGuTok - 1) / kGuTok;
    }
    const bool have = warp_wait(&full[idx], (s / S) & 1, &s_abort, a.flag);
    const unsigned char *st = stage_base + (size_t)idx * stage_bytes;
    const unsigned char *sgb = st + scl_off + ((lr0 * sclb) & 15);
    const unsigned char *sub = st + scl_off + span_stride + ((lr1 * sclb) & 15);
    for (int grp = 0; grp < ngroups; ++grp, ++it) {
      const int nt = min(kGuTok, cnt - grp * kGuTok);
      const bool last = grp == ngroups - 1;
      if (ngroups > 1 || new_expert) {
        // token of slot g of this group; the decision to reload depends only on shared
        // data, so all compute warps take it together
        const int pr = pairs_of_expert<kGuTok>(R.ids, n, R.act_e[ai], grp * kGuTok, lane);
        mypair = __shfl_sync(0xFFFFFFFFu, pr, g & 7);
        // activation row of slot g: token (gate/up) or h row of the slot (down)
        const int tok = g >= nt ? -1
                        : (MODE == 0 ? (int)(mypair / K) : R.act_off[ai] + grp * kGuTok + g);
        const bool reload = __any_sync(0xFFFFFFFFu, tok != loaded_tok);
        if (reload) {
          loaded_tok = tok;
          // pass 1: largest magnitude of token g over the whole row (all compute warps)
          float mx = 0.f;
          if (tok >= 0) {
#pragma unroll
            for (int m = 0; m < MC; ++m) {
              const int c = cw + CW * m;
              if (c < nchunk && c * 128 + 32 * t < Kd) {
                uint4 v[4];
                mx = fmaxf(mx, load_bf16x32(arow + (int64_t)tok * Kd + c * 128 + 32 * t, v));
              }
            }
          }
          mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
          if (t == 0) smax[cw * kGuTok + g] = mx;
          named_sync(1, nthreads_c);
          float mm = 0.f;
          for (int w = 0; w < CW; ++w) mm = fmaxf(mm, smax[w * kGuTok + g]);
          const int p = prescale_exponent(mm);
          pscale = exp2i(-p);
          const float sp = exp2i(p);
#pragma unroll
          for (int m = 0; m < MC; ++m) {
            const int c = cw + CW * m;
            if (tok >= 0 && c < nchunk && c * 128 + 32 * t < Kd) {
              uint4 v[4];
              load_bf16x32(arow + (int64_t)tok * Kd + c * 128 + 32 * t, v);
              to_f16x32(v, sp, xr[m]);
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) xr[m][i] = 0u;
            }
          }
          named_sync(1, nthreads_c);   // smax is rewritten by the next reload
        }
      }
      // partial dot products over this warp's chunks: per M-tile mt, d[0..3] = tile rows
      // (16 mt + g, 16 mt + 8 + g) x tokens (2t, 2t+1) as the m16n8 accumulator layout has
      // them; two chains per M-tile for latency
      float d0[MT][4], d1[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) d0[mt][i] = d1[mt][i] = 0.f;
      if (have) {
#pragma unroll
        for (int m = 0; m < MC; ++m) {
          const int c = cw + CW * m;
          if (c >= nchunk) break;
          const bool lv = c * 128 + 32 * t < Kd;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            // tile rows R0 = 16 mt + g and R1 = R0 + 8; their scales sit in the run of the
            // half (first HALF rows, or the rest) that holds them
            const int R0 = 16 * mt + g, R1 = R0 + 8;
            const unsigned char *s0 = 16 * mt >= HALF ? sub + (R0 - HALF) * sclb : sgb + R0 * sclb;
            const unsigned char *s1 =
                16 * mt + 8 >= HALF ? sub + (R1 - HALF) * sclb : sgb + R1 * sclb;
            uint4 wg = make_uint4(0u, 0u, 0u, 0u), wu = wg;
            uint32_t sg = 0u, su = 0u;
            if (lv) {
              wg = *reinterpret_cast<const uint4 *>(st + R0 * rstride + c * 64 + 16 * t);
              wu = *reinterpret_cast<const uint4 *>(st + R1 * rstride + c * 64 + 16 * t);
              sg = *reinterpret_cast<const unsigned short *>(s0 + c * 8 + 2 * t);
              su = *reinterpret_cast<const unsigned short *>(s1 + c * 8 + 2 * t);
            }
            // block scales as f16 pairs: blocks 2t (elements 0..15 of the lane) and 2t+1
            const uint32_t sgh = e4m3x2_to_f16x2(sg), suh = e4m3x2_to_f16x2(su);
            const uint32_t Sg[2] = {__byte_perm(sgh, 0, 0x1010), __byte_perm(sgh, 0, 0x3232)};
            const uint32_t Su[2] = {__byte_perm(suh, 0, 0x1010), __byte_perm(suh, 0, 0x3232)};
            const uint32_t wgw[4] = {wg.x, wg.y, wg.z, wg.w};
            const uint32_t wuw[4] = {wu.x, wu.y, wu.z, wu.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {          // word q: elements 8q..8q+7, MMAs 2q, 2q+1
              uint32_t hg[4], hu[4];
              e2m1x8_to_f16x2x4(wgw[q], hg);
              e2m1x8_to_f16x2x4(wuw[q], hu);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                hg[k] = hmul2_u32(hg[k], Sg[q >> 1]);
                hu[k] = hmul2_u32(hu[k], Su[q >> 1]);
              }
              // MMA 2q: elements 8q..8q+3; MMA 2q+1: elements 8q+4..8q+7
              mma_16816_f16(d0[mt], hg[0], hu[0], hg[1], hu[1], xr[m][4 * q], xr[m][4 * q + 1]);
              mma_16816_f16(d1[mt], hg[2], hu[2], hg[3], hu[3], xr[m][4 * q + 2],
                            xr[m][4 * q + 3]);
            }
          }
        }
      }
      if (last) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[idx]);   // this warp is done reading the stage
      }
      const int sl = it % kRedSlots;
      if (it >= kRedSlots) warp_wait(&rfree[sl], ((it / kRedSlots) - 1) & 1, &s_abort, a.flag);
      // this warp's partials: M-tile mt, token tk, row r at mt * 128 + tk * 16 + r
      float *rb = red + (size_t)sl * RF + cw * 128 * MT;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        rb[mt * 128 + (2 * t) * 16 + g] = d0[mt][0] + d1[mt][0];
        rb[mt * 128 + (2 * t + 1) * 16 + g] = d0[mt][1] + d1[mt][1];
        rb[mt * 128 + (2 * t) * 16 + 8 + g] = d0[mt][2] + d1[mt][2];
        rb[mt * 128 + (2 * t + 1) * 16 + 8 + g] = d0[mt][3] + d1[mt][3];
      }
      if (cw == 0 && t == 0) {
        red[(size_t)sl * RF + CW * 128 * MT + g] = pscale;
        red[(size_t)sl * RF + CW * 128 * MT + kGuTok + g] = __int_as_float(mypair);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rfull[sl]);
    }
  }
}

// ================================================================== down + combine (one token)
// CTA c owns output rows [n0, n0 + nb) (nb <= kDownRows) for every active expert; a stage
// holds srows of them (one expert's rows in ceil(nb / srows) stages).  Warp 0 produces; warps 1..CW compute, each taking whole rows (row r
// of a stage belongs to warp r % CW), with lane l owning the 16-byte units l, l + 32, ... of
// the packed row (32 elements, two blocks, each), so a row's dot product needs only the
// warp's own shuffle reduction.  The h rows of all slots arrive in shared memory with one
// bulk copy and are scaled to f16 once.  The per-pair results stay in shared memory (yk)
// and are combined in ascending k at the end.
template <int UPL, int CW, int S>
__global__ void __launch_bounds__(32 * (CW + 1))
    gemv_down_kernel(MoeArgs a, uint32_t stage_bytes, int nb, int srows) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t H = a.H, I = a.I, K = a.K;
  const int n = (int)K;   // one token: pair k is slot-routed directly
  const int E = (int)a.E;
  constexpr int RPW = (kDownRows + CW - 1) / CW;   // rows of a stage per warp
  static_assert((RPW & (RPW - 1)) == 0 && RPW <= 32, "rows per warp must be a power of two");
  const Smem L = smem_layout(S, stage_bytes, CW, 0, n, E, n * nb, (uint32_t)(n * I * 2));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint64_t *empty = full + S;
  uint64_t *hbar = empty + S;
  unsigned char *stage_base = smem + L.stages;
  float *pss = reinterpret_cast<float *>(smem + L.smax);   // [n] 2^-p of each slot
  CtaRoute R{reinterpret_cast<int *>(smem + L.ids), reinterpret_cast<int *>(smem + L.act_e),
             reinterpret_cast<int *>(smem + L.act_off), reinterpret_cast<int *>(smem + L.misc)};
  int *hist = reinterpret_cast<int *>(smem + L.hist);
  int *slot_of = reinterpret_cast<int *>(smem + L.slot);
  int *run = reinterpret_cast<int *>(smem + L.run);
  float *yk = reinterpret_cast<float *>(smem + L.yk);
  uint4 *hsm = reinterpret_cast<uint4 *>(smem + L.hpre);   // [n][I/8]: bf16, then scaled f16

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    mbar_init(hbar, 1);
    mbar_init_fence();
  }
  // The ids were complete before the gate/up kernel let this grid start; reading them
  // (and the weights) before griddepcontrol.wait overlaps this prologue with its tail.
  cta_route(a.ids, n, E, a.map, R, hist);
  const int n_act = *R.n_act;
  if (warp == 1) warp_slots(R.ids, n, hist, R.act_off, n_act, run, slot_of, lane);
  __syncthreads();

  const int n0 = blockIdx.x * nb;
  const int n1 = min((int)H, n0 + nb);
  const int nr = max(0, n1 - n0);   // rows of this CTA (per expert)
  const uint32_t rowb = (uint32_t)(I / 2), sclb = (uint32_t)(I / 16);
  const int cpe = nr > 0 ? (nr + srows - 1) / srows : 0;   // stages per expert
  const int n_stages = n_act * cpe;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      for (; s < n_stages; ++s) {
        const int e = R.act_e[s / cpe];
        const int q0 = (s % cpe) * srows;           // first row of the stage (from n0)
        const int nq = min(srows, nr - q0);
        const int idx = s % S;
        if (s >= S && (*(volatile int *)&s_abort || !mbar_wait(&empty[idx], ((s / S) - 1) & 1))) {
          if (!*(volatile int *)&s_abort) report_timeout(a.flag);
          *(volatile int *)&s_abort = 1;
          break;
        }
        unsigned char *st = stage_base + (size_t)idx * stage_bytes;
        const int64_t row = (int64_t)e * H + n0 + q0;
        const int64_t ls = (int64_t)(n0 + q0) * sclb;
        const uint32_t span = (uint32_t)(((ls + nq * sclb + 15) & ~15ll) - (ls & ~15ll));
        mbar_arrive_expect_tx(&full[idx], (uint32_t)nq * rowb + span);
        bulk_g2s(st, a.w_dn + row * rowb, nq * rowb, &full[idx]);
        bulk_g2s_span(st + srows * rowb, a.s_dn + (int64_t)e * H * sclb, ls, nq * sclb, &full[idx]);
      }
      const int issued = s;
      for (int t = max(0, issued - S); t < issued; ++t)
        if (!mbar_wait(&full[t % S], (t / S) & 1)) report_timeout(a.flag);
    }
    return;
  }

  // ------------------------------------------------ compute warps
  const int cw = warp - 1;
  const int nthreads_c = CW * 32;
  pdl_wait();   // h is written by the gate/up kernel
  pdl_launch_dependents();
  // The gate/up grid is complete: its work counters are zero again (its last CTA reset
  // them); rewriting them here keeps them zero even after a gate/up launch that failed.
  if (blockIdx.x == 0 && cw == 0 && lane == 0) {
    a.work[0] = 0;
    a.work[1] = 0;
  }
  const int n_valid = R.act_off[n_act];   // slots 0..n_valid-1 are the rows of h in use
  if (cw == 0 && lane == 0 && n_valid > 0) {
    const uint32_t bytes = (uint32_t)((int64_t)n_valid * I * 2);
    mbar_arrive_expect_tx(hbar, bytes);
    bulk_g2s(hsm, a.h, bytes, hbar);
  }
  if (n_valid > 0) warp_wait(hbar, 0, &s_abort, a.flag);
  // Scale each slot by an exact power of two into f16 (warp cw takes slots cw, cw + CW, ...),
  // stored unit-transposed: 16-byte piece i of unit u (32 elements) goes to index i * U + u, so
  // the per-stage reloads below read consecutive 16-byte pieces across the lanes.  Lane l
  // reads pieces l, l + 32, ... (consecutive across the warp), and each group of 8 lanes
  // writes 8 consecutive transposed pieces, so neither side has bank conflicts.
  const int U = (int)(I / 32);   // 16-byte units per packed row = 64-byte units per h row
  for (int sl = cw; sl < n_valid; sl += CW) {
    uint4 *row = hsm + (size_t)sl * (4 * U);
    uint4 v[4 * UPL];
    float mm = 0.f;
#pragma unroll
    for (int j = 0; j < 4 * UPL; ++j) {
      const int pc = lane + 32 * j;   // piece in natural order: unit pc / 4, index pc % 4
      v[j] = pc < 4 * U ? row[pc] : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t w4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) mm = fmaxf(mm, fmaxf(fabsf(bf16_lo(w4[k])), fabsf(bf16_hi(w4[k]))));
    }
    mm = warp_max(mm);   // also orders every lane's reads before the writes below
    const int p = prescale_exponent(mm);
    const float sp = exp2i(p);
#pragma unroll
    for (int j = 0; j < 4 * UPL; ++j) {
      const int pc = lane + 32 * j;
      if (pc < 4 * U) {
        const uint4 q = v[j];
        row[(pc & 3) * U + (pc >> 2)] = make_uint4(f16x2_rn(bf16_lo(q.x) * sp, bf16_hi(q.x) * sp),
                                                   f16x2_rn(bf16_lo(q.y) * sp, bf16_hi(q.y) * sp),
                                                   f16x2_rn(bf16_lo(q.z) * sp, bf16_hi(q.z) * sp),
                                                   f16x2_rn(bf16_lo(q.w) * sp, bf16_hi(q.w) * sp));
      }
    }
    if (lane == 0) pss[sl] = exp2i(-p);
    __syncwarp();
  }
  named_sync(1, nthreads_c);

  for (int s = 0; s < n_stages; ++s) {
    const int idx = s % S;
    const int ai = s / cpe;
    const int q0 = (s % cpe) * srows;   // first row of the stage (from n0)
    const int nq = min(srows, nr - q0);
    const int slot0 = R.act_off[ai];
    const int cnt = R.act_off[ai + 1] - slot0;   // > 1 only for a repeated expert id
    const float g = __ldg(a.g_dn + R.act_e[ai]);
    const bool have = warp_wait(&full[idx], (s / S) & 1, &s_abort, a.flag);
    const unsigned char *st = stage_base + (size_t)idx * stage_bytes;
    const unsigned char *sbase = st + srows * rowb + (((int64_t)(n0 + q0) * sclb) & 15);
    for (int c = 0; c < cnt; ++c) {
      const int slot = slot0 + c;
      uint32_t xh[UPL][16];
      const uint4 *hrow = hsm + (size_t)slot * (4 * U);
#pragma unroll
      for (int k = 0; k < UPL; ++k) {
        const int u = lane + 32 * k;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = u < U ? hrow[i * U + u] : make_uint4(0u, 0u, 0u, 0u);
          xh[k][4 * i] = v.x;
          xh[k][4 * i + 1] = v.y;
          xh[k][4 * i + 2] = v.z;
          xh[k][4 * i + 3] = v.w;
        }
      }
      float flat[RPW];
#pragma unroll
      for (int i = 0; i < RPW; ++i) flat[i] = 0.f;
      if (have) {
        // two rows at a time (independent chains); a missing second row re-reads the first
#pragma unroll
        for (int i = 0; i < RPW; i += 2) {
          const int ra = cw + i * CW;
          if (ra >= nq) break;   // warp-uniform
          const int rb = ra + CW < nq ? ra + CW : ra;
          float acc_a = 0.f, acc_b = 0.f;
#pragma unroll
          for (int k = 0; k < UPL; ++k) {
            const int u = lane + 32 * k;
            if (u < U) {
              const uint4 qa = *reinterpret_cast<const uint4 *>(st + (size_t)ra * rowb + 16 * u);
              const uint4 qb = *reinterpret_cast<const uint4 *>(st + (size_t)rb * rowb + 16 * u);
              const uint32_t sa = e4m3x2_to_f16x2(
                  *reinterpret_cast<const unsigned short *>(sbase + (size_t)ra * sclb + 2 * u));
              const uint32_t sb = e4m3x2_to_f16x2(
                  *reinterpret_cast<const unsigned short *>(sbase + (size_t)rb * sclb + 2 * u));
              const float a0 = dot16(qa.x, qa.y, &xh[k][0]);
              const float b0 = dot16(qb.x, qb.y, &xh[k][0]);
              const float a1 = dot16(qa.z, qa.w, &xh[k][8]);
              const float b1 = dot16(qb.z, qb.w, &xh[k][8]);
              acc_a = fmaf(a1, f16_hi(sa), fmaf(a0, f16_lo(sa), acc_a));
              acc_b = fmaf(b1, f16_hi(sb), fmaf(b0, f16_lo(sb), acc_b));
            }
          }
          flat[i] = acc_a;
          if (i + 1 < RPW) flat[i + 1] = acc_b;
        }
      }
      if (c == cnt - 1) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[idx]);   // this warp is done reading the stage
      }
      const float tot = warp_reduce_many<RPW>(flat, lane);
      constexpr int SH = 5 - Log2<RPW>::value;
      const int r = cw + (lane >> SH) * CW;
      if ((lane & ((1 << SH) - 1)) == 0 && r < nq) yk[(size_t)slot * nb + q0 + r] = tot * g * pss[slot];
    }
  }
  named_sync(2, nthreads_c);   // every y of this CTA is in yk
  // combine in ascending k: out[n0 + o] = sum_k w[k] * y(slot(k))[o]
  const int ctid = threadIdx.x - 32;
  for (int o = ctid; o < nr; o += nthreads_c) {
    float acc = 0.f;
    for (int k = 0; k < K; ++k) {
      const int sl = slot_of[k];
      if (sl >= 0) acc += yk[(size_t)sl * nb + o] * __ldg(a.w + k);
    }
    if (a.out_f32)
      a.out_f32[n0 + o] = acc;
    else
      a.out[n0 + o] = __float2bfloat16_rn(acc);
  }
}

template <int NT, int P, int S>
int launch_gateup_cfg(const MoeArgs &a, cudaStream_t s, int ctas_per_sm) {
  const int CW = (int)ceil_div(a.H, 1024);
  const uint32_t stage_bytes = (uint32_t)(2 * P * (a.H / 2) + 2 * span_bytes(P * (a.H / 16)));
  const int n = (int)(a.T * a.K);
  const Smem L = smem_layout(S, stage_bytes, CW, 2 * P * NT, n, (int)a.E, 0);
  // one wave of resident CTAs that pull row chunks from a counter until none are left
  const int fit = resident_blocks(gemv_gateup_kernel<NT, P, S>, 32 * (CW + 2), L.total);
  if (fit <= 0) return fit < 0 ? NVFP4_ECUDA : NVFP4_ESHAPE;
  return launch_pdl(gemv_gateup_kernel<NT, P, S>, dim3(num_sms() * min(ctas_per_sm, fit)),
                    dim3(32 * (CW + 2)), L.total, s, a, stage_bytes);
}

template <int MODE, int S, int MC>
int launch_mma_cfg(const MoeArgs &a, cudaStream_t s) {
  const int n = (int)(a.T * a.K);
  const GuSmem L = gu_smem_layout(S, gu_stage_bytes(MODE == 0 ? a.H : a.I, 16 * gu_mtiles(MODE)),
                                  n, (int)a.E, gu_red_floats(MODE));
  const int fit = resident_blocks(gemv_mma_kernel<MODE, S, MC>, 32 * (kGuWarps + 1 + kGuFinal), L.total);
  if (fit <= 0) return fit < 0 ? NVFP4_ECUDA : NVFP4_ESHAPE;
  return launch_pdl(gemv_mma_kernel<MODE, S, MC>, dim3(num_sms()), dim3(32 * (kGuWarps + 1 + kGuFinal)),
                    L.total, s, a);
}

// Three stages when they fit in shared memory, else two (deeper rings measured no faster:
// with one bulk copy per 8 rows the stream keeps up).
template <int MODE>
int launch_mma(const MoeArgs &a, cudaStream_t s) {
  const int n = (int)(a.T * a.K);
  const uint32_t sb = gu_stage_bytes(MODE == 0 ? a.H : a.I, 16 * gu_mtiles(MODE));
  const bool three = gu_smem_layout(3, sb, n, (int)a.E, gu_red_floats(MODE)).total <= 227u * 1024u;
  // one chunk per warp covers a reduction of 16 * 128 = 2048 (the down projection at
  // I <= 2048): fewer registers held for the activations
  if ((MODE == 0 ? a.H : a.I) <= 16 * 128)
    return three ? launch_mma_cfg<MODE, 3, 1>(a, s) : launch_mma_cfg<MODE, 2, 1>(a, s);
  return three ? launch_mma_cfg<MODE, 3, kGuMaxChunks>(a, s)
               : launch_mma_cfg<MODE, 2, kGuMaxChunks>(a, s);
}

template <int UPL, int CW, int S>
int launch_down_cfg(const MoeArgs &a, cudaStream_t s, int ctas_per_sm) {
  const int n = (int)(a.T * a.K);
  // enough CTAs for the GPU, and at most kDownRows rows per CTA (one stage per expert)
  const int64_t want = max64((int64_t)num_sms() * ctas_per_sm, ceil_div(a.H, kDownRows));
  const int nb = (int)ceil_div(a.H, want);
  const int64_t ctas = ceil_div(a.H, nb);
  const int srows = (int)ceil_div(nb, kDownSplit);   // rows per stage
  const uint32_t stage_bytes =
      align_up((uint32_t)(srows * (a.I / 2)) + span_bytes(srows * (a.I / 16)), 128);
  const Smem L = smem_layout(S, stage_bytes, CW, 0, n, (int)a.E, n * nb, (uint32_t)(n * a.I * 2));
  const int fit = resident_blocks(gemv_down_kernel<UPL, CW, S>, 32 * (CW + 1), L.total);
  if (fit <= 0) return fit < 0 ? NVFP4_ECUDA : NVFP4_ESHAPE;
  return launch_pdl(gemv_down_kernel<UPL, CW, S>, dim3((unsigned)ctas), dim3(32 * (CW + 1)),
                    L.total, s, a, stage_bytes, nb, srows);
}

}  // namespace

bool gemv_supported(int64_t T, int64_t H, int64_t I, int64_t K) {
  if (T * K > kGemvMaxPairs) return false;
  if (T == 1)   // CUDA-core kernels: gate/up lanes own 32 elements of a row (6 warps), down
                // lanes up to three 32-element units
    return H <= 1024 * kMaxConsumerWarps && I <= 512 * kMaxConsumerWarps;
  const int64_t max_k = (int64_t)kGuWarps * kGuMaxChunks * 128;   // mma kernels
  return H <= max_k && I <= max_k;
}

// One token: the CUDA-core kernels (the combine is fused into the down kernel).  More
// tokens: the mma.sync kernels, which serve up to 8 tokens of an expert per MMA, and a
// separate combine.
bool gemv_fused_combine(int64_t T) { return T == 1; }

int launch_gemv_gateup(const MoeArgs &a, cudaStream_t s) {
  if (gemv_fused_combine(a.T))
    return launch_gateup_cfg<1, kPairs, kStages>(a, s, NVFP4_GEMV_CTAS_PER_SM);
  return launch_mma<0>(a, s);
}

int launch_gemv_down(const MoeArgs &a, cudaStream_t s) {
  if (gemv_fused_combine(a.T)) {   // one token: lanes own ceil(I / 1024) 16-byte units
    const int c = NVFP4_GEMV_DOWN_CTAS_PER_SM;
    if (a.I <= 1024) return launch_down_cfg<1, kDownWarps, kDownStages>(a, s, c);
    if (a.I <= 2048) return launch_down_cfg<2, kDownWarps, kDownStages>(a, s, c);
    return launch_down_cfg<3, kDownWarps, kDownStages>(a, s, c);
  }
  return launch_mma<1>(a, s);
}

}  // namespace nvfp4
