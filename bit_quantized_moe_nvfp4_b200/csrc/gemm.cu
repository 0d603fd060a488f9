// gemm.cu -- tensor-core grouped GEMM path of the NVFP4 MoE layer (tcgen05, sm_100a).
//
// Page "GLM-5-NVFP4-MTP", "Model Description": NVFP4 experts (4-bit values, one FP8 scale
// per 16 elements), 256 experts, 8 active per token.  With many tokens per expert each
// projection is a dense contraction per expert, run on the tensor cores:
//
//   gather:  xs[r] = x[token of routed pair r]           (pairs in expert order)
//   gate/up: D = W_gu[e] (rows j0..j0+63 gate, same rows up) . xs[slots of e]^T
//            h[slot, j] = bf16( silu(g_gu*D_gate) * g_gu*D_up )
//   down:    D = W_dn[e] (128 rows) . h[slots of e]^T
//            y[slot, n] = w[pair] * g_dn * D
//   combine (combine.cu): out[t] = bf16( sum over k of y[slot(t, k)] )
//
// One persistent CTA per SM walks the tiles (expert, 256-slot n-tile, 128-row m-tile) with
// warp-specialised roles:
//   warp 0     TMA producer: packed weight rows (2 boxes of 64 rows x 32 bytes) and the
//              activation tile (256 rows x 64 bf16, 128-byte swizzle) per 64-wide K step;
//   warp 1     allocates TMEM and issues tcgen05.mma (M=128, N<=256, K=16, fp32 in TMEM);
//   warps 2-5  dequantize: one weight row per thread, E2M1 x E4M3 -> bf16 (exact: at most 6
//              significant bits) written into the K-major SW128 operand tile;
//   warps 6-9  epilogue: tcgen05.ld of the accumulator, global scale, SwiGLU or routing
//              weight, stores.
// Accumulators are double-buffered in TMEM (2 x 256 columns), so the epilogue of one tile
// overlaps the main loop of the next.  The weights sit on M ("swap AB") because experts get
// anywhere from 0 to thousands of tokens: the token count only changes N.
#include <cuda.h>

#include "moe.cuh"
#include "tcgen05.cuh"

namespace nvfp4 {

namespace {

constexpr int BM = 128;          // weight rows per tile
constexpr int BN = 256;          // token slots per tile (largest N of one MMA)
constexpr int BK = 64;           // reduction elements per stage (128-byte bf16 rows)
constexpr int kS = 4;            // stages of packed weights + activation tiles
constexpr int kSA = 2;           // dequantized weight tiles
constexpr int kThreads = 320;    // 10 warps
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kBBytes = BN * BK * 2;     // 32 KB
constexpr uint32_t kABytes = BM * BK * 2;     // 16 KB
constexpr uint32_t kPBytes = BM * BK / 2;     // 4 KB packed
constexpr uint32_t kSmemB = 0;
constexpr uint32_t kSmemA = kSmemB + kS * kBBytes;
constexpr uint32_t kSmemP = kSmemA + kSA * kABytes;
constexpr uint32_t kSmemBars = kSmemP + kS * kPBytes;
constexpr uint32_t kSmemMisc = kSmemBars + 8 * (2 * kS + 2 * kSA + 4);
constexpr uint32_t kSmemTotal = kSmemMisc + 16 + 1024;   // + alignment slack

struct GemmParams {
  MoeArgs a;
  int mode;                 // 0: gate/up + SwiGLU -> h;  1: down -> y
  int K;                    // reduction length (H for gate/up, I for down)
  int m_tiles;              // m tiles per expert
  const uint8_t *scales;    // E4M3 block scales of the weights
  const float *gscale;      // per-expert global scales
};

struct TileInfo {
  int e;        // expert
  int mt;       // m tile
  int slot0;    // first slot (row of xs / h / y) of the n tile
  int nvalid;   // slots of this expert in the n tile (1..BN)
};

// Tile index -> (expert, n tile, m tile).  tile_prefix lists, for the active experts in
// ascending order, the number of n tiles before each.
__device__ __forceinline__ TileInfo tile_info(const GemmParams &p, int tile, int n_act) {
  const int ntg = tile / p.m_tiles;
  TileInfo t;
  t.mt = tile % p.m_tiles;
  int lo = 0, hi = n_act - 1;
  while (lo < hi) {  // last a with tile_prefix[a] <= ntg
    const int mid = (lo + hi + 1) >> 1;
    if (p.a.tile_prefix[mid] <= ntg)
      lo = mid;
    else
      hi = mid - 1;
  }
  t.e = p.a.active[lo];
  const int nloc = ntg - p.a.tile_prefix[lo];
  t.slot0 = p.a.offsets[t.e] + nloc * BN;
  t.nvalid = min(BN, p.a.counts[t.e] - nloc * BN);
  return t;
}

__device__ __forceinline__ int round16(int v) { return (v + 15) & ~15; }

// ------------------------------------------------------------------ dequantize one row
// 64 E2M1 codes (32 bytes) with 4 E4M3 block scales -> 64 bf16 in the K-major SW128 tile.
__device__ __forceinline__ void dequant_row(const uint4 (&q)[2], uint32_t scales4, unsigned char *a_tile,
                                            int arow) {
  const uint32_t words[8] = {q[0].x, q[0].y, q[0].z, q[0].w, q[1].x, q[1].y, q[1].z, q[1].w};
  const uint32_t s01 = e4m3x2_to_f16x2(scales4 & 0xFFFFu);
  const uint32_t s23 = e4m3x2_to_f16x2(scales4 >> 16);
  unsigned char *row = a_tile + (arow >> 3) * 1024 + (arow & 7) * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c) {          // 16-byte output chunk c = elements 8c..8c+7
    const uint32_t sb = (c < 4) ? ((c < 2) ? __byte_perm(s01, 0, 0x1010) : __byte_perm(s01, 0, 0x3232))
                                : ((c < 6) ? __byte_perm(s23, 0, 0x1010) : __byte_perm(s23, 0, 0x3232));
    uint32_t h[4];
    e2m1x8_to_f16x2x4(words[c], h);
    uint32_t o[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      // q * s is exact in f16 and in bf16 (at most 6 significant bits, within range)
      __half2 v = __hmul2(*reinterpret_cast<__half2 *>(&h[p]), *reinterpret_cast<const __half2 *>(&sb));
      const float2 f = __half22float2(v);
      o[p] = pack_bf16x2(f.x, f.y);
    }
    *reinterpret_cast<uint4 *>(row + ((c ^ (arow & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ------------------------------------------------------------------ the GEMM kernel
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                const __grid_constant__ CUtensorMap tmap_b, GemmParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem =
      smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);   // 1024-byte aligned
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kSmemBars);
  uint64_t *empty = full + kS;
  uint64_t *afull = empty + kS;
  uint64_t *aempty = afull + kSA;
  uint64_t *accfull = aempty + kSA;      // [2]
  uint64_t *accempty = accfull + 2;      // [2]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kSmemMisc);
  int *abort = reinterpret_cast<int *>(smem + kSmemMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const MoeArgs &a = p.a;

  if (threadIdx.x == 0) {
    *abort = 0;
    for (int s = 0; s < kS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < kSA; ++s) {
      mbar_init(&afull[s], 4);
      mbar_init(&aempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&accfull[s], 1);
      mbar_init(&accempty[s], 4);
    }
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  pdl_wait();   // routing tables (and the activations) come from earlier kernels
  const int n_act = *a.n_active;
  const int total_tiles = n_act > 0 ? a.tile_prefix[n_act] * p.m_tiles : 0;
  const int kblocks = p.K / BK;
  const int64_t I = a.I, H = a.H;

  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
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
      for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
        const TileInfo t = tile_info(p, tile, n_act);
        int row0, row1;   // first rows of the two 64-row boxes of packed weights
        if (p.mode == 0) {
          row0 = (int)((int64_t)t.e * 2 * I + t.mt * 64);
          row1 = (int)(row0 + I);
        } else {
          row0 = (int)((int64_t)t.e * H + t.mt * BM);
          row1 = row0 + 64;
        }
        for (int kb = 0; kb < kblocks; ++kb, ++kg) {
          const int s = kg % kS;
          if (kg >= kS && !wait(&empty[s], ((kg / kS) - 1) & 1)) break;
          if (*(volatile int *)abort) break;
          mbar_arrive_expect_tx(&full[s], kPBytes + kBBytes);
          unsigned char *pk = smem + kSmemP + s * kPBytes;
          tma_load_2d(pk, &tmap_w, kb * (BK / 2), row0, &full[s]);
          tma_load_2d(pk + 64 * (BK / 2), &tmap_w, kb * (BK / 2), row1, &full[s]);
          tma_load_2d(smem + kSmemB + s * kBBytes, &tmap_b, kb * BK, t.slot0, &full[s]);
        }
        if (*(volatile int *)abort) break;
      }
      // copies into this CTA's shared memory must land before it can exit
      for (int t = max(0, kg - kS); t < kg; ++t) mbar_wait(&full[t % kS], (t / kS) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int kg = 0, tc = 0;
      for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++tc) {
        const TileInfo t = tile_info(p, tile, n_act);
        const int acc = tc & 1;
        if (tc >= 2 && !wait(&accempty[acc], ((tc >> 1) - 1) & 1)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        const uint32_t idesc = idesc_bf16_f32(BM, max(16, round16(t.nvalid)));
        for (int kb = 0; kb < kblocks; ++kb, ++kg) {
          const int s = kg % kS, sa = kg % kSA;
          const bool ok = wait(&full[s], (kg / kS) & 1) && wait(&afull[sa], (kg / kSA) & 1);
          tc_fence_after();
          if (ok) {
            const uint32_t a_addr = smem_u32(smem + kSmemA + sa * kABytes);
            const uint32_t b_addr = smem_u32(smem + kSmemB + s * kBBytes);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_bf16(d_tmem, smem_desc_sw128(a_addr + 32 * kk), smem_desc_sw128(b_addr + 32 * kk),
                        idesc, kb > 0 || kk > 0);
          }
          umma_commit(&empty[s]);
          umma_commit(&aempty[sa]);
        }
        umma_commit(&accfull[acc]);
      }
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------------- dequantize
    const int dt = threadIdx.x - 64;            // packed row of the tile handled here
    int kg = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileInfo t = tile_info(p, tile, n_act);
      int64_t wrow;
      int arow;
      bool valid = true;
      if (p.mode == 0) {
        const int jj = dt & 63;
        wrow = (int64_t)t.e * 2 * I + (dt < 64 ? 0 : I) + t.mt * 64 + jj;
        arow = 2 * jj + (dt < 64 ? 0 : 1);       // gate j at row 2j, up j at row 2j+1
      } else {
        const int64_t n = (int64_t)t.mt * BM + dt;
        valid = n < H;
        wrow = (int64_t)t.e * H + n;
        arow = dt;
      }
      const uint8_t *srow = p.scales + wrow * (p.K / 16);
      uint32_t sc_next = valid ? __ldg(reinterpret_cast<const uint32_t *>(srow)) : 0u;
      for (int kb = 0; kb < kblocks; ++kb, ++kg) {
        const int s = kg % kS, sa = kg % kSA;
        const uint32_t sc = sc_next;
        if (kb + 1 < kblocks && valid)
          sc_next = __ldg(reinterpret_cast<const uint32_t *>(srow) + kb + 1);
        bool ok = wait(&full[s], (kg / kS) & 1);
        if (kg >= kSA) ok = wait(&aempty[sa], ((kg / kSA) - 1) & 1) && ok;
        if (ok) {
          const uint4 *src = reinterpret_cast<const uint4 *>(smem + kSmemP + s * kPBytes + dt * (BK / 2));
          uint4 q[2] = {src[0], src[1]};
          if (!valid) q[0] = q[1] = make_uint4(0, 0, 0, 0);
          dequant_row(q, sc, smem + kSmemA + sa * kABytes, arow);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[sa]);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;                     // TMEM lane quarter of this warp
    const int m = q * 32 + lane;                // accumulator row (TMEM lane)
    int tc = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++tc) {
      const TileInfo t = tile_info(p, tile, n_act);
      const int acc = tc & 1;
      const bool ok = wait(&accfull[acc], (tc >> 1) & 1);
      tc_fence_after();
      const float g = __ldg(p.gscale + t.e);
      const int ncols = round16(t.nvalid);
      for (int c0 = 0; ok && c0 < ncols; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + c0, v);
        if (p.mode == 0) {
          const int64_t j = (int64_t)t.mt * 64 + (m >> 1);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float val = __uint_as_float(v[c]) * g;
            const float other = __shfl_xor_sync(0xFFFFFFFFu, val, 1);
            if (!(lane & 1) && c0 + c < t.nvalid) {
              const float hv = silu_f32(val) * other;       // val = gate, other = up
              a.h[(int64_t)(t.slot0 + c0 + c) * I + j] = __float2bfloat16_rn(hv);
            }
          }
        } else {
          const int64_t n = (int64_t)t.mt * BM + m;
          const int sl = t.slot0 + c0 + lane;
          const float wl = (c0 + lane < t.nvalid) ? __ldg(a.w + a.perm[sl]) * g : 0.f;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float wc = __shfl_sync(0xFFFFFFFFu, wl, c);
            if (n < H && c0 + c < t.nvalid)
              a.y[(int64_t)(t.slot0 + c0 + c) * H + n] = __uint_as_float(v[c]) * wc;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[acc]);
    }
  }

  // all roles are done: release tensor memory
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ gather
// xs[r] = x[perm[r] / K] for the routed pairs (one warp per row, 16-byte copies).
__global__ void __launch_bounds__(256) gather_kernel(MoeArgs a) {
  pdl_wait();
  const int64_t H = a.H, K = a.K;
  const int n_valid = a.offsets[a.E];
  const int vec = (int)(H / 8);
  const int64_t warps = (int64_t)gridDim.x * 8;
  for (int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); r < n_valid; r += warps) {
    const int64_t t = a.perm[r] / K;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.x + t * H);
    uint4 *dst = reinterpret_cast<uint4 *>(a.xs + r * H);
    for (int i = threadIdx.x & 31; i < vec; i += 32) dst[i] = __ldg(src + i);
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D tiled map over a row-major [rows, cols] array.
int make_map(CUtensorMap *m, CUtensorMapDataType type, int elem_bytes, const void *base,
             uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
             CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return NVFP4_ECUDA;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, type, 2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ECUDA;
}

int launch_gemm(const MoeArgs &a, int mode, cudaStream_t s) {
  GemmParams p;
  p.a = a;
  p.mode = mode;
  const int64_t rows_per_expert = mode == 0 ? 2 * a.I : a.H;
  p.K = (int)(mode == 0 ? a.H : a.I);
  p.m_tiles = (int)(mode == 0 ? a.I / 64 : ceil_div(a.H, BM));
  p.scales = mode == 0 ? a.s_gu : a.s_dn;
  p.gscale = mode == 0 ? a.g_gu : a.g_dn;
  CUtensorMap tw, tb;
  // packed weights: [E * rows_per_expert, K/2] bytes, boxes of 64 rows x 32 bytes
  if (make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, mode == 0 ? a.w_gu : a.w_dn,
               (uint64_t)(p.K / 2), (uint64_t)(a.E * rows_per_expert), BK / 2, 64,
               CU_TENSOR_MAP_SWIZZLE_NONE))
    return NVFP4_ECUDA;
  // activations: [T*K + pad, K] bf16, boxes of BN rows x 64 elements, 128-byte swizzle
  const uint64_t brows = (uint64_t)(a.T * a.K + kGatherPadRows);
  if (make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, mode == 0 ? (const void *)a.xs
                                                                     : (const void *)a.h,
               (uint64_t)p.K, brows, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return NVFP4_ECUDA;
  cudaError_t e =
      cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  int dev = 0, sms = kNumSMs;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return launch_pdl(gemm_kernel, dim3(sms), dim3(kThreads), kSmemTotal, s, tw, tb, p);
}

}  // namespace

int gemm_tile_n() { return BN; }

int launch_gemm_gateup(const MoeArgs &a, cudaStream_t s) {
  const int64_t rows = a.T * a.K;
  int64_t blocks = ceil_div(rows, 8);
  if (blocks > kNumSMs * 8) blocks = kNumSMs * 8;
  if (int st = launch_pdl(gather_kernel, dim3((unsigned)blocks), dim3(256), 0, s, a)) return st;
  return launch_gemm(a, 0, s);
}

int launch_gemm_down(const MoeArgs &a, cudaStream_t s) { return launch_gemm(a, 1, s); }

}  // namespace nvfp4
