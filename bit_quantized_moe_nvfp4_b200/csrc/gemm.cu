// gemm.cu -- tensor-core grouped GEMM path of the NVFP4 MoE layer (tcgen05, sm_100a).
//
// Page "GLM-5-NVFP4-MTP", "Model Description": NVFP4 experts (4-bit values, one FP8 scale
// per 16 elements), 256 experts, 8 active per token.  With many tokens per expert each
// projection is a dense contraction per expert, run on the tensor cores:
//
//   gather:  xs[r] = f16(x[token of pair r] * 2^p_r)   (pairs in expert order, exact
//            per-row power-of-two scale, xscale[r] = 2^-p_r)
//   gate/up: D = W_gu[e] (rows j0..j0+63 gate, same rows up) . xs[slots of e]^T   (f16 MMA)
//            h[slot, j] = bf16( silu(g_gu*xscale*D_gate) * g_gu*xscale*D_up )
//   down:    D = W_dn[e] (128 rows) . h[slots of e]^T                          (bf16 MMA)
//            y[slot, n] = w[pair] * g_dn * D
//   combine (combine.cu): out[t] = bf16( sum over k of y[slot(t, k)] )
//
// One persistent CTA per SM walks the tiles (expert, 192-slot n-tile, 128-row m-tile) with
// warp-specialised roles:
//   warp 0     TMA producer: packed weight rows (2 boxes of 64 rows x 64 bytes) and the
//              activation tile (2 boxes of 192 rows x 64 elements, 128-byte swizzle) per
//              128-wide K step, into a 3-stage ring;
//   warp 1     allocates TMEM and issues tcgen05.mma (M=128, N<=192, K=16, fp32 in TMEM)
//              with the weight operand read from TMEM and the activations from shared memory;
//   warps 2-9  dequantize: half a weight row per thread, E2M1 x E4M3 -> f16 (gate/up) or
//              bf16 (down), exact either way (at most 6 significant bits), stored straight
//              into the thread's TMEM lane (tcgen05.st), so the dequantized operand never
//              touches shared memory;
//   warps 10-13 epilogue: tcgen05.ld of the accumulator, global scale, SwiGLU or routing
//              weight, stores.
// Accumulators are double-buffered in TMEM (2 x 192 columns, next to two 64-column weight
// operand slots), so the epilogue of one tile overlaps the main loop of the next.  The weights sit on M ("swap AB") because experts get
// anywhere from 0 to thousands of tokens: the token count only changes N.
#include <cuda.h>

#include "moe.cuh"
#include "tcgen05.cuh"

namespace nvfp4 {

namespace {

// Pipeline depth, tile sizes and dequant width (compile-time tunables; defaults measured on
// B200: a 128-wide K step issues 8 MMAs per barrier round trip, which is what lets the
// single issuing thread keep the tensor pipe busy).
#ifndef NVFP4_GEMM_STAGES
#define NVFP4_GEMM_STAGES 3
#endif
#ifndef NVFP4_GEMM_BN
#define NVFP4_GEMM_BN 192
#endif
#ifndef NVFP4_GEMM_A_SLOTS
#define NVFP4_GEMM_A_SLOTS 2
#endif
#ifndef NVFP4_GEMM_DEQUANT_WARPS
#define NVFP4_GEMM_DEQUANT_WARPS 8
#endif
#ifndef NVFP4_GEMM_BK
#define NVFP4_GEMM_BK 128
#endif
constexpr int BM = 128;          // weight rows per tile (TMEM lanes)
constexpr int BN = NVFP4_GEMM_BN;   // token slots per tile (MMA N, multiple of 16)
constexpr int BK = NVFP4_GEMM_BK;   // reduction elements per stage (64 or 128)
constexpr int kBoxes = BK / 64;     // 64-element (128-byte) activation boxes per stage
static_assert(BK == 64 || BK == 128, "BK: 64 or 128");
constexpr int kS = NVFP4_GEMM_STAGES;           // stages: packed weights + activation tile
constexpr int kSA = NVFP4_GEMM_A_SLOTS;         // weight operand slots in TMEM
constexpr int kDQW = NVFP4_GEMM_DEQUANT_WARPS;  // 4 (full rows) or 8 (half rows)
constexpr int kWarpEpi = 2 + kDQW;              // first of the 4 epilogue warps
constexpr int kThreads = 32 * (kWarpEpi + 4);
static_assert(kDQW == 4 || kDQW == 8, "dequant warps: 4 or 8");

// Tensor memory: two fp32 accumulators of BN columns, then kSA weight operands of BK/2
// columns (BK 16-bit values of a row per lane) -- 2*192 + 2*64 = 512 columns.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemA = 2 * BN;
constexpr uint32_t kACols = BK / 2;
static_assert(kTmemA + kSA * kACols <= kTmemCols, "TMEM budget");

constexpr uint32_t kBoxBytes = BN * 128;     // one 64-element activation box (128-byte swizzle)
constexpr uint32_t kBBytes = kBoxes * kBoxBytes;
static_assert(kBoxBytes % 1024 == 0, "swizzled tiles start on 1024-byte boundaries");
constexpr uint32_t kPBytes = BM * BK / 2;     // packed weights (4 or 8 KB)
constexpr int kSB = BK / 16;                  // block-scale bytes per row per stage
constexpr uint32_t kSmemB = 0;
constexpr uint32_t kSmemP = kSmemB + kS * kBBytes;
// epilogue staging: two buffers of one 32-column chunk of the output tile (down: 32 slots x
// 128 rows fp32 = 16 KB; gate/up: 32 slots x 64 bf16 = 4 KB), written to HBM by TMA stores
constexpr uint32_t kOutBufBytes = 32 * BM * 4;
constexpr uint32_t kSmemOut = kSmemP + kS * kPBytes;
constexpr uint32_t kSmemBars = kSmemOut + 2 * kOutBufBytes;
constexpr uint32_t kSmemMisc = kSmemBars + 8 * (2 * kS + 2 * kSA + 4);
constexpr uint32_t kSmemTotal = kSmemMisc + 16 + 1024;   // + alignment slack
static_assert(kSmemTotal <= 227 * 1024, "shared memory budget");

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

// v[i] for a runtime i < N without dynamic register indexing.
template <int N>
__device__ __forceinline__ float pick(const float (&v)[N], int i) {
  float r = v[0];
#pragma unroll
  for (int k = 1; k < N; ++k)
    if (i == k) r = v[k];
  return r;
}

// silu(z) = z / (1 + e^-z) with the fast exponential and division (a few ulp of fp32; h is
// rounded to bf16 right after).  For z below about -88, e^-z is infinite and the quotient 0.
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// ------------------------------------------------------------------ dequantize
// NW packed words (8 E2M1 codes each) with their NW/2 block scales (one byte per 16
// elements, low bytes first) -> 4*NW packed 16-bit pairs, each the exact product e2m1*e4m3:
//   f16:  the hardware E2M1 -> f16 convert, then one f16 multiply by the scale.
//   bf16: the f16 magnitude bits shifted right by 3 read as bf16 are |q| * 2^-112 (the exponent
//         field widens from 5 to 8 bits; q has one mantissa bit, so nothing is lost), one
//         bf16 multiply by s * 2^112 (exact, below 2^121) gives |q| * s, and the sign bit is
//         copied back.  This keeps the conversion on the integer pipes.
template <bool F16, int NW>
__device__ __forceinline__ void dequant_words(const uint32_t (&words)[NW], uint32_t scales,
                                              uint32_t (&out)[4 * NW]) {
  uint32_t sb[NW / 2];   // per block: the scale in both halves, f16 or bf16(s * 2^112)
#pragma unroll
  for (int b = 0; b < NW / 2; b += 2) {
    const uint32_t s2 = e4m3x2_to_f16x2((scales >> (8 * b)) & 0xFFFFu);
    const uint32_t sh[2] = {__byte_perm(s2, 0, 0x1010), __byte_perm(s2, 0, 0x3232)};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (b + k >= NW / 2) break;
      if (F16) {
        sb[b + k] = sh[k];
      } else {
        const float sv = f16_lo(sh[k]) * 5.192296858534828e33f;   // s * 2^112
        sb[b + k] = pack_bf16x2(sv, sv);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < NW; ++c) {
    uint32_t h[4];
    e2m1x8_to_f16x2x4(words[c], h);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t s2 = sb[c >> 1];
      if (F16) {
        __half2 v = __hmul2(*reinterpret_cast<__half2 *>(&h[p]), *reinterpret_cast<const __half2 *>(&s2));
        out[4 * c + p] = *reinterpret_cast<uint32_t *>(&v);
      } else {
        uint32_t mag = (h[p] >> 3) & 0x0FFF0FFFu;
        __nv_bfloat162 v = __hmul2(*reinterpret_cast<__nv_bfloat162 *>(&mag),
                                   *reinterpret_cast<const __nv_bfloat162 *>(&s2));
        out[4 * c + p] = *reinterpret_cast<uint32_t *>(&v) | (h[p] & 0x80008000u);
      }
    }
  }
}

// ------------------------------------------------------------------ the GEMM kernel
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                const __grid_constant__ CUtensorMap tmap_b,
                const __grid_constant__ CUtensorMap tmap_out, GemmParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem =
      smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);   // 1024-byte aligned
  // Stage s holds packed weights P[s] and the activation tile B[s]; the weight operand of
  // K step kg lives in TMEM slot kg % kSA.
  //   full[s]    TMA bytes of P[s] and B[s] have landed            (producer -> dequant)
  //   freeb[s]   the MMAs reading B[s] are done                    (MMA commit -> producer)
  //   afull[sa]  TMEM weight slot sa is written (P, B landed)      (dequant -> MMA)
  //   afree[sa]  the MMAs reading TMEM slot sa are done            (MMA commit -> dequant)
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kSmemBars);
  uint64_t *freeb = full + kS;
  uint64_t *afull = freeb + kS;
  uint64_t *afree = afull + kSA;
  uint64_t *accfull = afree + kSA;       // [2]
  uint64_t *accempty = accfull + 2;      // [2]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kSmemMisc);
  int *abort = reinterpret_cast<int *>(smem + kSmemMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const MoeArgs &a = p.a;

  if (threadIdx.x == 0) {
    *abort = 0;
    for (int s = 0; s < kS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&freeb[s], 1);
    }
    for (int s = 0; s < kSA; ++s) {
      mbar_init(&afull[s], kDQW);
      mbar_init(&afree[s], 1);
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
  const int kblocks = (p.K + BK - 1) / BK;   // a last half stage (K % 128 == 64) reads zeros
  const int64_t I = a.I, H = a.H;

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
          if (kg >= kS && !wait(&freeb[s], ((kg / kS) - 1) & 1)) break;
          if (*(volatile int *)abort) break;
          mbar_arrive_expect_tx(&full[s], kPBytes + kBBytes);
          unsigned char *pk = smem + kSmemP + s * kPBytes;
          tma_load_2d(pk, &tmap_w, kb * (BK / 2), row0, &full[s]);
          tma_load_2d(pk + 64 * (BK / 2), &tmap_w, kb * (BK / 2), row1, &full[s]);
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_2d(smem + kSmemB + s * kBBytes + bx * kBoxBytes, &tmap_b, kb * BK + 64 * bx,
                        t.slot0, &full[s]);
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
        const int nmma = max(16, round16(t.nvalid));
        const uint32_t idesc = p.mode == 0 ? idesc_f16_f32(BM, nmma) : idesc_bf16_f32(BM, nmma);
        for (int kb = 0; kb < kblocks; ++kb, ++kg) {
          const int s = kg % kS, sa = kg % kSA;
          const bool ok = wait(&afull[sa], (kg / kSA) & 1);   // implies full[s]
          tc_fence_after();
          if (ok) {
            const uint32_t a_tmem = tmem_base + kTmemA + sa * kACols;
            const uint64_t db = smem_desc_sw128(smem_u32(smem + kSmemB + s * kBBytes));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)   // K=16: 8 TMEM columns, 32 bytes of a B box
              umma_ts(d_tmem, a_tmem + 8 * kk,
                      db + (uint64_t)((kk / 4) * (kBoxBytes >> 4) + 2 * (kk % 4)), idesc,
                      kb > 0 || kk > 0);
          }
          umma_commit(&freeb[s]);
          umma_commit(&afree[sa]);
        }
        umma_commit(&accfull[acc]);
      }
    }
  } else if (warp < kWarpEpi) {
    // ---------------------------------------------------------------- dequantize
    // Warp w writes TMEM lanes 32*(w%4)..+31: lane L holds weight-operand row L.  With 8
    // warps, the second four write the upper half of each row's 64 elements.
    constexpr int kPerRow = kDQW / 4;            // threads per row (1 or 2)
    constexpr int NW = BK / 8 / kPerRow;         // packed words per thread per step
    static_assert(NW == 4 || NW == 8, "one tcgen05.st of 16 or 32 columns per step");
    const int q = warp & 3;
    const int part = (warp - 2) / 4;             // 0, or 1 for the second four warps
    const int L = q * 32 + lane;                 // operand row = TMEM lane
    int kg = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileInfo t = tile_info(p, tile, n_act);
      int64_t wrow;
      int prow;            // row of the packed tile feeding operand row L
      bool valid = true;
      if (p.mode == 0) {
        const int jj = L >> 1;                   // gate j at row 2j, up j at row 2j+1
        prow = (L & 1) ? 64 + jj : jj;
        wrow = (int64_t)t.e * 2 * I + ((L & 1) ? I : 0) + t.mt * 64 + jj;
      } else {
        const int64_t n = (int64_t)t.mt * BM + L;
        valid = n < H;
        prow = L;
        wrow = (int64_t)t.e * H + n;
      }
      // Block scales of this row: BK/16 bytes per K step (one or two 32-bit words), fetched
      // 16 bytes at a time, two groups ahead.  Rows whose scale run is not 16-byte aligned
      // take 4-byte loads; words past the end of the row read as 0.
      constexpr int kWS = kSB / 4;             // scale words per stage
      constexpr int kSPG = 4 / kWS;            // stages per 16-byte group
      const uint8_t *srow = p.scales + wrow * (p.K / 16);
      const int n_words = p.K / 64;
      const bool wide = (p.K % 256) == 0;
      auto group = [&](int g) -> uint4 {
        if (!valid || 4 * g >= n_words) return make_uint4(0, 0, 0, 0);
        if (wide) return __ldg(reinterpret_cast<const uint4 *>(srow) + g);
        const uint32_t *w = reinterpret_cast<const uint32_t *>(srow) + 4 * g;
        const int left = n_words - 4 * g;
        return make_uint4(__ldg(w), left > 1 ? __ldg(w + 1) : 0u, left > 2 ? __ldg(w + 2) : 0u,
                          left > 3 ? __ldg(w + 3) : 0u);
      };
      uint4 g0 = group(0), g1 = group(1), g2 = group(2);
      for (int kb = 0; kb < kblocks; ++kb, ++kg) {
        const int s = kg % kS, sa = kg % kSA;
        if (kb > 0 && kb % kSPG == 0) {
          g0 = g1;
          g1 = g2;
          g2 = group(kb / kSPG + 2);
        }
        const int w4 = (kb % kSPG) * kWS + (kWS == 2 ? part : 0);
        const uint32_t sc = w4 == 0 ? g0.x : (w4 == 1 ? g0.y : (w4 == 2 ? g0.z : g0.w));
        bool ok = wait(&full[s], (kg / kS) & 1);
        if (kg >= kSA) ok = wait(&afree[sa], ((kg / kSA) - 1) & 1) && ok;
        tc_fence_after();
        uint32_t w[NW];
        // The packed rows arrive with the 64-byte swizzle: 16-byte chunk c of row r sits at
        // chunk c ^ ((r >> 1) & 3), so the rows read at one column spread over the banks.
        const unsigned char *prow_base = smem + kSmemP + s * kPBytes + prow * (BK / 2);
        const int sw = (prow >> 1) & 3;
#pragma unroll
        for (int i = 0; i < NW; i += 4) {
          const int chunk = (part * NW + i) / 4;
          const uint4 v = *reinterpret_cast<const uint4 *>(prow_base + 16 * (chunk ^ sw));
          w[i] = v.x;
          w[i + 1] = v.y;
          w[i + 2] = v.z;
          w[i + 3] = v.w;
        }
        if (!valid || !ok)
#pragma unroll
          for (int i = 0; i < NW; ++i) w[i] = 0u;
        const uint32_t scp = kWS == 2 ? sc : sc >> (8 * (NW / 2) * part);   // this part's scales
        uint32_t o[4 * NW];
        if (p.mode == 0)
          dequant_words<true, NW>(w, scp, o);
        else
          dequant_words<false, NW>(w, scp, o);
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + kTmemA + sa * kACols +
                               part * (kACols / kPerRow);
        if (NW == 8)
          tmem_st32(taddr, *reinterpret_cast<uint32_t(*)[32]>(o));
        else
          tmem_st16(taddr, *reinterpret_cast<uint32_t(*)[16]>(o));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[sa]);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;                     // TMEM lane quarter of this warp (the four
                                                // epilogue warps are consecutive)
    const int m = q * 32 + lane;                // accumulator row (TMEM lane)
    int tc = 0;
    int nchunk_out = 0;                         // chunks sent through the staging buffers
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++tc) {
      const TileInfo t = tile_info(p, tile, n_act);
      const int acc = tc & 1;
      const bool ok = wait(&accfull[acc], (tc >> 1) & 1);
      tc_fence_after();
      const float g = __ldg(p.gscale + t.e);
      const int ncols = round16(t.nvalid);
      // per-column factors of the tile (slot c0 + lane of each 32-column chunk), all loaded
      // before the first accumulator read: 2^-p (gate/up) or the routing weight (down)
      constexpr int kChunks = (BN + 31) / 32;
      float colf[kChunks];
      {
        int pr[kChunks];
#pragma unroll
        for (int ch = 0; ch < kChunks; ++ch) {
          const int col = 32 * ch + lane;
          pr[ch] = (col < t.nvalid && p.mode == 1) ? __ldg(a.perm + t.slot0 + col) : 0;
        }
#pragma unroll
        for (int ch = 0; ch < kChunks; ++ch) {
          const int col = 32 * ch + lane;
          colf[ch] = col >= t.nvalid ? 0.f
                     : (p.mode == 0 ? a.xscale[t.slot0 + col] : __ldg(a.w + pr[ch])) * g;
        }
      }
      for (int c0 = 0; ok && c0 < ncols; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + c0, v);
        const float cf = pick<kChunks>(colf, c0 >> 5);
        // A chunk whose 32 slots all belong to the tile goes out through shared memory and
        // one TMA store; a partial chunk (the expert's last few slots) is stored directly,
        // so no row of the next expert is touched.
        const bool full_chunk = c0 + 32 <= t.nvalid;
        unsigned char *ob = smem + kSmemOut + (size_t)(nchunk_out & 1) * kOutBufBytes;
        if (full_chunk) {
          // the store that last read this buffer (two chunks ago) is done: see below
          named_sync(3, 128);
        }
        if (p.mode == 0) {
          const int jl = q * 16 + (lane >> 1);     // column of h within the m tile (0..63)
          const int64_t j = (int64_t)t.mt * 64 + jl;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float val = __uint_as_float(v[c]) * __shfl_sync(0xFFFFFFFFu, cf, c);
            const float other = __shfl_xor_sync(0xFFFFFFFFu, val, 1);
            const __nv_bfloat16 hv = __float2bfloat16_rn(silu_fast(val) * other);  // gate, up
            if (!(lane & 1)) {
              if (full_chunk)
                reinterpret_cast<__nv_bfloat16 *>(ob)[c * 64 + jl] = hv;
              else if (c0 + c < t.nvalid)
                a.h[(int64_t)(t.slot0 + c0 + c) * I + j] = hv;
            }
          }
        } else {
          const int64_t n = (int64_t)t.mt * BM + m;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float yv = __uint_as_float(v[c]) * __shfl_sync(0xFFFFFFFFu, cf, c);
            if (full_chunk)
              reinterpret_cast<float *>(ob)[c * BM + m] = yv;
            else if (n < H && c0 + c < t.nvalid)
              a.y[(int64_t)(t.slot0 + c0 + c) * H + n] = yv;
          }
        }
        if (full_chunk) {
          fence_proxy_async_smem();   // generic writes -> visible to the TMA engine
          named_sync(3, 128);
          if (warp == kWarpEpi && lane == 0) {
            if (p.mode == 0)
              tma_store_2d(&tmap_out, t.mt * 64, t.slot0 + c0, ob);
            else
              tma_store_2d(&tmap_out, t.mt * BM, t.slot0 + c0, ob);
            bulk_commit_group();
            bulk_wait_group_read<1>();   // the other buffer may be rewritten
          }
          ++nchunk_out;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[acc]);
    }
    if (warp == kWarpEpi && lane == 0) bulk_wait_group_all();   // every TMA store is done
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
// xs[r] = f16(x[perm[r] / K] * 2^p_r), xscale[r] = 2^-p_r, for the routed pairs: one warp
// per row, 16-byte accesses; the row is read twice (largest magnitude, then convert), the
// second time from cache.
__global__ void __launch_bounds__(256) gather_kernel(MoeArgs a) {
  pdl_wait();
  const int64_t H = a.H, K = a.K;
  const int n_valid = a.offsets[a.E];
  const int vec = (int)(H / 8);
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * 8;
  for (int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); r < n_valid; r += warps) {
    const int64_t t = a.perm[r] / K;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.x + t * H);
    uint4 *dst = reinterpret_cast<uint4 *>(a.xs + r * H);
    float m = 0.f;
    for (int i = lane; i < vec; i += 32) {
      const uint4 v = __ldg(src + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[k])), fabsf(bf16_hi(w[k]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int p = prescale_exponent(m);
    const float sc = exp2i(p);
    for (int i = lane; i < vec; i += 32) {
      const uint4 v = __ldg(src + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        __half2 hv = __floats2half2_rn(bf16_lo(w[k]) * sc, bf16_hi(w[k]) * sc);
        o[k] = *reinterpret_cast<uint32_t *>(&hv);
      }
      dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (lane == 0) a.xscale[r] = exp2i(-p);
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ host side
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
  // packed weights: [E * rows_per_expert, K/2] bytes, boxes of 64 rows x BK/2 bytes with the
  // 64-byte swizzle (the dequantize warps' reads undo it)
  static_assert(BK / 2 == 64, "the 64-byte swizzle spans exactly one packed row");
  if (make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, mode == 0 ? a.w_gu : a.w_dn,
               (uint64_t)(p.K / 2), (uint64_t)(a.E * rows_per_expert), BK / 2, 64,
               CU_TENSOR_MAP_SWIZZLE_64B))
    return NVFP4_ECUDA;
  // activations: [T*K + pad, K] f16 (gate/up) or bf16 (down), boxes of BN rows x 64
  // elements, 128-byte swizzle
  const uint64_t brows = (uint64_t)(a.T * a.K + kGatherPadRows);
  if (make_map(&tb, mode == 0 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
               2, mode == 0 ? (const void *)a.xs : (const void *)a.h,
               (uint64_t)p.K, brows, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return NVFP4_ECUDA;
  // outputs for the epilogue's TMA stores: h [T*K + pad, I] bf16 in boxes of 32 slots x 64,
  // or y [T*K, H] fp32 in boxes of 32 slots x 128
  CUtensorMap to;
  if (mode == 0) {
    if (make_map(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.h, (uint64_t)a.I, brows, 64, 32,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
      return NVFP4_ECUDA;
  } else {
    if (make_map(&to, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.y, (uint64_t)a.H,
                 (uint64_t)(a.T * a.K), BM, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
      return NVFP4_ECUDA;
  }
  cudaError_t e =
      cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  int dev = 0, sms = kNumSMs;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return launch_pdl(gemm_kernel, dim3(sms), dim3(kThreads), kSmemTotal, s, tw, tb, to, p);
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
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
