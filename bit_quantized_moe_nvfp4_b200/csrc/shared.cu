// shared.cu -- the shared expert: a dense BF16 SwiGLU MLP that every token passes through,
// added to the routed experts' output before the layer output is rounded to bf16.
//
// Page "GLM-5-NVFP4-MTP", "What's quantized": only the routed experts' gate, up and down
// projections are NVFP4 and the rest of the model stays BF16; a page on the same model
// family lists the shared experts among its BF16 tensors.  For every token t:
//   h_s[t, j] = bf16( silu(Wg[j] . x_t) * (Wu[j] . x_t) )         j < Is
//   out[t, n] = bf16( routed[t, n] + Wd[n] . h_s[t] )              n < H
// with Wg / Wu the rows 0..Is-1 / Is..2Is-1 of w_gu [2Is, H] and Wd = w_dn [H, Is]; the
// products of bf16 values are exact and the sums fp32.  routed is the fp32 sum over the
// token's routed experts (moe_nvfp4_forward_ep's partial), or absent.
//
// Two implementations of one function:
//  * T <= kGemvMaxT tokens: the 3 * Is * H weights are the whole cost (75 MB at H = 6144,
//    Is = 2048).  Warps stream weight rows with 16-byte loads against the tokens held in
//    shared memory (gate/up: four warps per row pair, down: one per row) and reduce across
//    their lanes.
//  * more tokens: one tcgen05 GEMM per projection.  A CTA tile is 128 weight rows (gate/up:
//    64 gate rows and the matching 64 up rows, so the SwiGLU stays inside the tile) by 256
//    tokens.  Both operands come by TMA into a 4-stage ring of 128-byte-swizzled shared
//    memory; one thread issues the MMAs (K = 16 each, 64 per stage) into one of two TMEM
//    accumulators while four epilogue warps drain the other.
#include <algorithm>

#include "moe.cuh"
#include "tcgen05.cuh"

namespace nvfp4 {
namespace {

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

constexpr int kGemvMaxT = 8;
constexpr int kGemvThreads = 256;

struct SharedArgs {
  const __nv_bfloat16 *x;      // [T, H]
  const __nv_bfloat16 *w_gu;   // [2 Is, H]
  const __nv_bfloat16 *w_dn;   // [H, Is]
  __nv_bfloat16 *h;            // [T, Is]  SwiGLU output (workspace)
  const float *routed;         // [T, H]   fp32 routed sum, or null
  __nv_bfloat16 *out;          // [T, H]
  int32_t *flag;               // error bits (may be null)
  int64_t T, H, Is;
};

// acc + (8 bf16 of w) . (8 bf16 of x), fp32, in element order.
__device__ __forceinline__ float dot8(uint4 w, uint4 x, float acc) {
  acc = fmaf(bf16_lo(w.x), bf16_lo(x.x), acc);
  acc = fmaf(bf16_hi(w.x), bf16_hi(x.x), acc);
  acc = fmaf(bf16_lo(w.y), bf16_lo(x.y), acc);
  acc = fmaf(bf16_hi(w.y), bf16_hi(x.y), acc);
  acc = fmaf(bf16_lo(w.z), bf16_lo(x.z), acc);
  acc = fmaf(bf16_hi(w.z), bf16_hi(x.z), acc);
  acc = fmaf(bf16_lo(w.w), bf16_lo(x.w), acc);
  acc = fmaf(bf16_hi(w.w), bf16_hi(x.w), acc);
  return acc;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// ------------------------------------------------------------------ few tokens (CUDA cores)
// Gate/up: the reduction of each row pair (gate row j, up row Is + j) is split over kSplit
// warps of one CTA, so a CTA of 8 warps takes 8 / kSplit row pairs per pass and every SM
// holds enough loads in flight; the tokens' x rows sit in shared memory.  The kSplit partial
// sums are added in warp order, then lane t < T of the finishing threads writes h[t, j].
constexpr int kSplit = 4;
template <int NT>
__global__ void __launch_bounds__(kGemvThreads) shared_gemv_gateup(SharedArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int kRowPairs = kGemvThreads / 32 / kSplit;   // row pairs per CTA pass
  __shared__ float part_sum[kRowPairs][kSplit][NT][2];
  uint4 *xs = reinterpret_cast<uint4 *>(smem);   // [T][H / 8]
  const int T = (int)a.T;
  const int64_t H = a.H, Is = a.Is;
  const int n8 = (int)(H / 8);
  const int per = n8 / kSplit;                   // 16-byte words of a row per warp
  pdl_wait();   // x may come from the previous kernel
  for (int i = threadIdx.x; i < T * n8; i += blockDim.x)
    xs[i] = __ldg(reinterpret_cast<const uint4 *>(a.x) + i);
  __syncthreads();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rp = warp / kSplit, part = warp % kSplit;
  for (int64_t j0 = (int64_t)blockIdx.x * kRowPairs; j0 < Is; j0 += (int64_t)gridDim.x * kRowPairs) {
    const int64_t j = j0 + rp;
    float g[NT], u[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) g[t] = u[t] = 0.f;
    if (j < Is) {
      const uint4 *wg = reinterpret_cast<const uint4 *>(a.w_gu + j * H);
      const uint4 *wu = reinterpret_cast<const uint4 *>(a.w_gu + (Is + j) * H);
#pragma unroll 4
      for (int c = part * per + lane; c < (part + 1) * per; c += 32) {
        const uint4 vg = ldg_stream(wg + c), vu = ldg_stream(wu + c);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if (t < T) {
            const uint4 xv = xs[t * n8 + c];
            g[t] = dot8(vg, xv, g[t]);
            u[t] = dot8(vu, xv, u[t]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float gs = warp_sum(g[t]), us = warp_sum(u[t]);
      if (lane == 0) {
        part_sum[rp][part][t][0] = gs;
        part_sum[rp][part][t][1] = us;
      }
    }
    __syncthreads();
    if (threadIdx.x < kRowPairs * T) {
      const int r = threadIdx.x / T, t = threadIdx.x % T;
      if (j0 + r < Is) {
        float gv = 0.f, uv = 0.f;
#pragma unroll
        for (int p = 0; p < kSplit; ++p) {
          gv += part_sum[r][p][t][0];
          uv += part_sum[r][p][t][1];
        }
        a.h[t * Is + j0 + r] = __float2bfloat16_rn(silu_f32(gv) * uv);
      }
    }
    __syncthreads();
  }
}

// Down: warp w takes output rows n = w, w + warps, ...; the tokens' h rows sit in shared
// memory.  Lane t < T writes out[t, n] = bf16(routed[t, n] + sum).
template <int NT>
__global__ void __launch_bounds__(kGemvThreads) shared_gemv_down(SharedArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint4 *hs = reinterpret_cast<uint4 *>(smem);   // [T][Is / 8]
  const int T = (int)a.T;
  const int64_t H = a.H, Is = a.Is;
  const int n8 = (int)(Is / 8);
  pdl_wait();   // h comes from the gate/up kernel, routed from the routed layer before it
  for (int i = threadIdx.x; i < T * n8; i += blockDim.x)
    hs[i] = __ldcg(reinterpret_cast<const uint4 *>(a.h) + i);
  __syncthreads();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t n = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp; n < H; n += nwarps) {
    const uint4 *wd = reinterpret_cast<const uint4 *>(a.w_dn + n * Is);
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.f;
#pragma unroll 8
    for (int c = lane; c < n8; c += 32) {
      const uint4 v = ldg_stream(wd + c);
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (t < T) acc[t] = dot8(v, hs[t * n8 + c], acc[t]);
    }
    float mine = 0.f;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float s = warp_sum(acc[t]);
      if (lane == t) mine = s;
    }
    if (lane < T) {
      const float r = a.routed ? __ldcg(a.routed + lane * H + n) : 0.f;
      a.out[lane * H + n] = __float2bfloat16_rn(r + mine);
    }
  }
}

template <int NT>
int launch_gemv_pair(const SharedArgs &a, cudaStream_t s) {
  const int sms = num_sms();
  const size_t smem_gu = (size_t)a.T * a.H * 2, smem_dn = (size_t)a.T * a.Is * 2;
  if (smem_gu > 227 * 1024 || smem_dn > 227 * 1024) return NVFP4_ESHAPE;
  const int rg = resident_blocks(shared_gemv_gateup<NT>, kGemvThreads, smem_gu);
  const int rd = resident_blocks(shared_gemv_down<NT>, kGemvThreads, smem_dn);
  if (rg <= 0 || rd <= 0) return rg < 0 || rd < 0 ? NVFP4_ECUDA : NVFP4_ESHAPE;
  const int wpc = kGemvThreads / 32;
  const int64_t gg = min64(ceil_div(a.Is, wpc / kSplit), (int64_t)sms * rg);
  const int64_t gd = min64(ceil_div(a.H, wpc), (int64_t)sms * rd);
  if (int st = launch_pdl(shared_gemv_gateup<NT>, dim3((unsigned)gg), dim3(kGemvThreads), smem_gu,
                          s, a))
    return st;
  return launch_pdl(shared_gemv_down<NT>, dim3((unsigned)gd), dim3(kGemvThreads), smem_dn, s, a);
}

// ------------------------------------------------------------------ many tokens (tcgen05)
constexpr int DBM = 128;                        // weight rows per tile (TMEM lanes)
constexpr int DBN = 256;                        // tokens per tile (MMA N)
constexpr int DS = 4;                           // pipeline stages (64 reduction elements each)
constexpr uint32_t kDA = DBM * 128;             // weight tile per stage: 128 rows x 128 B
constexpr uint32_t kDB = DBN * 128;             // token tile per stage: 256 rows x 128 B
constexpr uint32_t kDStage = kDA + kDB;
constexpr uint32_t kDU = DS * kDStage;          // SwiGLU exchange: 64 up rows x 17 fp32
constexpr uint32_t kDUBytes = 64 * 17 * 4;
constexpr uint32_t kDBars = kDU + kDUBytes;
constexpr uint32_t kDMisc = kDBars + 8 * (2 * DS + 4);
constexpr uint32_t kDSmem = kDMisc + 16 + 1024;   // + alignment slack
constexpr int kDThreads = 192;                  // producer, MMA, 4 epilogue warps
static_assert(kDSmem <= 227 * 1024, "shared memory budget");
static_assert(kDA % 1024 == 0 && kDStage % 1024 == 0, "swizzled tiles on 1024-byte boundaries");

struct DenseParams {
  SharedArgs a;
  int mode;      // 0: gate/up + SwiGLU -> h;  1: down (+ routed) -> out
  int K;         // reduction length: H (gate/up) or Is (down), a multiple of 64
  int m_tiles, n_tiles;
};

__global__ void __launch_bounds__(kDThreads, 1)
    shared_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_b, DenseParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  //   full[s]      both tiles of stage s have landed      (TMA -> MMA)
  //   freeb[s]     the MMAs reading stage s are done      (MMA commit -> producer)
  //   accfull[b]   accumulator b holds a finished tile    (MMA commit -> epilogue)
  //   accempty[b]  the epilogue has read accumulator b    (4 epilogue warps -> MMA)
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kDBars);
  uint64_t *freeb = full + DS;
  uint64_t *accfull = freeb + DS;
  uint64_t *accempty = accfull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kDMisc);
  int *abort = reinterpret_cast<int *>(smem + kDMisc + 4);
  float *U = reinterpret_cast<float *>(smem + kDU);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SharedArgs &a = p.a;

  if (threadIdx.x == 0) {
    *abort = 0;
    for (int s = 0; s < DS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&freeb[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 2 * DBN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  pdl_wait();   // x, or h and the routed sum, come from the previous kernels
  const int total = p.m_tiles * p.n_tiles;
  const int kblocks = p.K / 64;
  const int64_t T = a.T, H = a.H, Is = a.Is;

  // Bounded wait; after any wait of the CTA has given up, later slow waits return at once.
  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    if (*(volatile int *)abort) return false;
    if (mbar_wait(bar, parity)) return true;
    *(volatile int *)abort = 1;
    report_timeout(a.flag);
    return false;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int kg = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
        for (int kb = 0; kb < kblocks; ++kb, ++kg) {
          const int s = kg % DS;
          if (kg >= DS && !wait(&freeb[s], ((kg / DS) - 1) & 1)) break;
          if (*(volatile int *)abort) break;
          mbar_arrive_expect_tx(&full[s], kDStage);
          unsigned char *A = smem + s * kDStage;
          if (p.mode == 0) {   // 64 gate rows, then the matching 64 up rows
            tma_load_2d(A, &tmap_w, kb * 64, mt * 64, &full[s]);
            tma_load_2d(A + kDA / 2, &tmap_w, kb * 64, (int)(Is + mt * 64), &full[s]);
          } else {
            tma_load_2d(A, &tmap_w, kb * 64, mt * DBM, &full[s]);
          }
          tma_load_2d(A + kDA, &tmap_b, kb * 64, nt * DBN, &full[s]);
        }
        if (*(volatile int *)abort) break;
      }
      // copies into this CTA's shared memory must land before it can exit
      for (int t = max(0, kg - DS); t < kg; ++t) mbar_wait(&full[t % DS], (t / DS) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int kg = 0, tc = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tc) {
        const int nt = tile / p.m_tiles;
        const int acc = tc & 1;
        if (tc >= 2 && !wait(&accempty[acc], ((tc >> 1) - 1) & 1)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * DBN;
        const int left = (int)min64(DBN, T - (int64_t)nt * DBN);
        const int nmma = max(16, (left + 15) & ~15);
        const uint32_t idesc = idesc_bf16_f32(DBM, nmma);
        for (int kb = 0; kb < kblocks; ++kb, ++kg) {
          const int s = kg % DS;
          const bool ok = wait(&full[s], (kg / DS) & 1);
          tc_fence_after();
          if (ok) {
            const uint64_t da = smem_desc_sw128(smem_u32(smem + s * kDStage));
            const uint64_t db = smem_desc_sw128(smem_u32(smem + s * kDStage + kDA));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)   // K = 16: 32 bytes along the 128-byte rows
              umma_bf16(d_tmem, da + 2 * kk, db + 2 * kk, idesc, kb > 0 || kk > 0);
          }
          umma_commit(&freeb[s]);
        }
        umma_commit(&accfull[acc]);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2-5)
    // Warp w reads TMEM lanes 32 (w % 4) .. +31: lane L is weight row L of the tile.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int tc = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tc) {
      const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
      const int acc = tc & 1;
      if (!wait(&accfull[acc], (tc >> 1) & 1)) break;
      tc_fence_after();
      const int64_t t0 = (int64_t)nt * DBN;
      const int ncols = (int)min64(DBN, T - t0);
      const uint32_t tb = tmem_base + acc * DBN + ((uint32_t)(q * 32) << 16);
      for (int c0 = 0; c0 < ncols; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tb + c0, v);
        if (p.mode == 0) {
          if (q >= 2) {   // up rows: hand them to the gate rows' threads
#pragma unroll
            for (int c = 0; c < 16; ++c) U[(row - 64) * 17 + c] = __uint_as_float(v[c]);
          }
          named_sync(1, 128);
          if (q < 2) {
            const int64_t j = (int64_t)mt * 64 + row;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int64_t t = t0 + c0 + c;
              if (t < T)
                a.h[t * Is + j] =
                    __float2bfloat16_rn(silu_f32(__uint_as_float(v[c])) * U[row * 17 + c]);
            }
          }
          named_sync(1, 128);
        } else {
          // The routed sums of the 16 tokens are all loaded before the first store: the
          // compiler cannot tell `routed` and `out` apart, so interleaving them would make
          // every load wait for the store before it.
          const int64_t n = (int64_t)mt * DBM + row;
          const bool nv = n < H;
          float r[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int64_t t = t0 + c0 + c;
            r[c] = (a.routed && nv && t < T) ? __ldcg(a.routed + t * H + n) : 0.f;
          }
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int64_t t = t0 + c0 + c;
            if (nv && t < T) a.out[t * H + n] = __float2bfloat16_rn(r[c] + __uint_as_float(v[c]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  pdl_launch_dependents();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * DBN);
  }
}

int launch_shared_gemm(const SharedArgs &a, int mode, cudaStream_t s) {
  DenseParams p;
  p.a = a;
  p.mode = mode;
  p.K = (int)(mode == 0 ? a.H : a.Is);
  p.m_tiles = (int)(mode == 0 ? a.Is / 64 : ceil_div(a.H, DBM));
  p.n_tiles = (int)ceil_div(a.T, DBN);
  CUtensorMap tw, tb;
  // weights [2 Is, H] (boxes of 64 rows) or [H, Is] (boxes of 128 rows), 64 elements wide
  if (make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, mode == 0 ? a.w_gu : a.w_dn,
               (uint64_t)p.K, (uint64_t)(mode == 0 ? 2 * a.Is : a.H), 64,
               mode == 0 ? 64 : DBM, CU_TENSOR_MAP_SWIZZLE_128B))
    return NVFP4_ECUDA;
  // tokens: x [T, H] or h [T, Is], boxes of 256 rows (rows past T read as zeros)
  if (make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
               mode == 0 ? (const void *)a.x : (const void *)a.h, (uint64_t)p.K,
               (uint64_t)a.T, 64, DBN, CU_TENSOR_MAP_SWIZZLE_128B))
    return NVFP4_ECUDA;
  if (resident_blocks(shared_gemm_kernel, kDThreads, kDSmem) <= 0) return NVFP4_ECUDA;
  const int total = p.m_tiles * p.n_tiles;
  const int grid = std::min(total, num_sms());
  return launch_pdl(shared_gemm_kernel, dim3(grid), dim3(kDThreads), kDSmem, s, tw, tb, p);
}

int launch_shared(const SharedArgs &a, cudaStream_t s) {
  if (a.T <= kGemvMaxT) {
    if (a.T <= 1) return launch_gemv_pair<1>(a, s);
    if (a.T <= 2) return launch_gemv_pair<2>(a, s);
    if (a.T <= 4) return launch_gemv_pair<4>(a, s);
    return launch_gemv_pair<8>(a, s);
  }
  if (int st = launch_shared_gemm(a, 0, s)) return st;
  return launch_shared_gemm(a, 1, s);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int check_shared(const __nv_bfloat16 *x, int64_t T, int64_t H, int64_t Is,
                 const __nv_bfloat16 *w_gu, const __nv_bfloat16 *w_dn, const float *routed,
                 const __nv_bfloat16 *out) {
  if (!x || !w_gu || !w_dn || !out || T <= 0 || H <= 0 || Is <= 0) return NVFP4_EINVAL;
  if (H % 64 || Is % 64 || H > 65536 || Is > 65536 || T >= (int64_t(1) << 31) / H)
    return NVFP4_ESHAPE;
  if (!aligned16(x) || !aligned16(w_gu) || !aligned16(w_dn) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(routed) & 3))
    return NVFP4_EINVAL;
  return NVFP4_OK;
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" size_t moe_nvfp4_shared_workspace_size(int64_t T, int64_t Is) {
  if (T <= 0 || Is <= 0) return 0;
  return align256((size_t)(T * Is * 2));
}

extern "C" int moe_nvfp4_shared_expert(const __nv_bfloat16 *x, int64_t T, int64_t H, int64_t Is,
                                       const __nv_bfloat16 *w_gu, const __nv_bfloat16 *w_dn,
                                       const float *routed, __nv_bfloat16 *out,
                                       void *workspace, size_t ws_bytes, cudaStream_t stream) {
  if (int st = check_shared(x, T, H, Is, w_gu, w_dn, routed, out)) return st;
  if (!workspace || !aligned16(workspace) || ws_bytes < moe_nvfp4_shared_workspace_size(T, Is))
    return NVFP4_EWORKSPACE;
  SharedArgs a = {x, w_gu, w_dn, static_cast<__nv_bfloat16 *>(workspace), routed, out, nullptr,
                  T, H, Is};
  return launch_shared(a, stream);
}

extern "C" size_t moe_nvfp4_layer_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E,
                                                 int64_t K, int64_t Is) {
  const size_t routed = moe_nvfp4_workspace_size(T, H, I, E, K);
  if (!routed || Is <= 0) return 0;
  return routed + align256((size_t)(T * H * 4)) + moe_nvfp4_shared_workspace_size(T, Is);
}

extern "C" int moe_nvfp4_layer(const __nv_bfloat16 *x, const float *router_logits, int64_t T,
                               int64_t H, int64_t I, int64_t E, int64_t K, const uint8_t *w_gu,
                               const uint8_t *s_gu, const float *g_gu, const uint8_t *w_dn,
                               const uint8_t *s_dn, const float *g_dn,
                               const __nv_bfloat16 *shared_gu, const __nv_bfloat16 *shared_dn,
                               int64_t Is, __nv_bfloat16 *out, int32_t *topk_ids_out,
                               float *topk_w_out, void *workspace, size_t ws_bytes, int path,
                               cudaStream_t stream) {
  if (!router_logits) return NVFP4_EINVAL;
  if (int st = check_shared(x, T, H, Is, shared_gu, shared_dn, nullptr, out)) return st;
  const size_t routed_bytes = moe_nvfp4_workspace_size(T, H, I, E, K);
  if (!routed_bytes) return NVFP4_EINVAL;
  if (!workspace || !aligned16(workspace) ||
      ws_bytes < moe_nvfp4_layer_workspace_size(T, H, I, E, K, Is))
    return NVFP4_EWORKSPACE;
  char *ws = static_cast<char *>(workspace);
  float *partial = reinterpret_cast<float *>(ws + routed_bytes);
  __nv_bfloat16 *hs =
      reinterpret_cast<__nv_bfloat16 *>(ws + routed_bytes + align256((size_t)(T * H * 4)));
  // the routed experts (router first), fp32, then the shared expert adds and rounds
  if (int st = forward_logits_partial(x, router_logits, T, H, I, E, K, w_gu, s_gu, g_gu, w_dn,
                                      s_dn, g_dn, partial, topk_ids_out, topk_w_out, workspace,
                                      routed_bytes, path, stream))
    return st;
  SharedArgs a = {x, shared_gu, shared_dn, hs, partial, out,
                  reinterpret_cast<int32_t *>(workspace), T, H, Is};
  return launch_shared(a, stream);
}
