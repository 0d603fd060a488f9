// w4a4.cu -- the routed-expert layer on the block-scaled FP4 tensor cores ("W4A4"): the
// activations are quantized to NVFP4 on the fly, and tcgen05.mma kind::mxf4nvf4 applies the
// weights' and the activations' E4M3 block scales inside the MMA.
//
// Page "GLM-5-NVFP4-MTP", "How to Run": the NVFP4 checkpoint is served with ModelOpt FP4
// quantization and FP4 MoE kernels.  The pages do not say how activations are scaled.  Here
// each activation row is quantized as a tensor of its own with the codec's arithmetic
// (quant.cuh): a token's x for gate/up, a routed pair's bf16 h for down.  That gives a dynamic
// per-row global scale g_row, one E4M3 scale per 16 elements and E2M1 codes.  Then
//   a[slot, j] = g_w[e] * g_row(slot) * sum over K of e2m1(W) e4m3(sW) e2m1(X) e4m3(sX)
// with the per-element products exact inside the MMA and fp32 accumulation.
//
// Data flow (one stream, each kernel launched with programmatic dependent launch):
//   route, n-tiles of 128 slots           -> routing tables
//   quantize each token's x row once      -> codes, scales and g per token
//   copy them into the padded slots        -> xq [P, H/2], scale atoms, g_x [P]
//   GEMM gate/up + SwiGLU                 -> h [T*K, I] bf16, slot order
//   quantize the h rows into padded slots -> hq [P, I/2], scale atoms, g_h [P]
//   GEMM down                             -> y [T*K, H] fp32 = w * g_dn * g_h * D
//   combine (combine.cu)                  -> out bf16
// Padded slots: each active expert's slots start on a multiple of 128 (its n-tiles are
// tile_prefix[a] .. tile_prefix[a+1]).  So an n-tile's activation rows and scale atoms are
// contiguous and aligned; rows past an expert's count are zero.
//
// Scale-factor layout, the tensor core's block-scaled operand format: one 512-byte atom per
// 128 rows and 64 elements along K.  Row r's four E4M3 scales (16 elements each) form the
// 32-bit word at byte 16 (r % 32) + 4 (r / 32).  tcgen05.cp .32x128b.warpx4 moves an atom to
// four TMEM columns, repeated in every lane quarter, so lane r finds its row's word in column
// r / 32.  The weights' scales are rearranged into atoms once (nvfp4_w4a4_prepare_scales);
// the activation quantizer writes atoms directly.
#include <algorithm>

#include "moe.cuh"
#include "quant.cuh"
#include "tcgen05.cuh"

namespace nvfp4 {
namespace {

constexpr int kPadN = 128;   // slots per n-tile (MMA N <= 128)

// silu(z) = z / (1 + e^-z) with the fast exponential and division (a few ulp of fp32; h is
// rounded to bf16 right after).  For z below about -88, e^-z is infinite and the quotient 0.
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

__host__ __device__ __forceinline__ int64_t round_up(int64_t v, int64_t m) {
  return (v + m - 1) / m * m;
}

// Byte offset of row r's scale for 16-element block b in a tensor of `cols` columns.
__host__ __device__ __forceinline__ int64_t atom_offset(int64_t r, int64_t b, int64_t cols) {
  return ((r / 128) * (cols / 64) + b / 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) / 32) + (b % 4);
}

// ------------------------------------------------------------------ weight scales -> atoms
// in: [n, rows, cols/16] row-major; out: [n][rows/128][cols/64][512].  With gate_rows = I > 0
// the tensor is a fused gate/up weight [2I, cols] and atom group m holds gate rows
// 64m..64m+63, then up rows I+64m..I+64m+63 (the rows of one GEMM tile).
__global__ void __launch_bounds__(256) swizzle_scales_kernel(const uint8_t *__restrict__ in,
                                                             int64_t n, int64_t rows,
                                                             int64_t cols, int64_t gate_rows,
                                                             uint8_t *__restrict__ out) {
  const int64_t kc = cols / 64, groups = rows / 128;
  const int64_t total = n * groups * kc * 128;   // one 4-byte word per (atom, row)
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i % 128, atom = i / 128;
    const int64_t c = atom % kc, grp = (atom / kc) % groups, t = atom / (kc * groups);
    const int64_t src = gate_rows ? (r < 64 ? 64 * grp + r : gate_rows + 64 * grp + (r - 64))
                                  : 128 * grp + r;
    const uint32_t word =
        *reinterpret_cast<const uint32_t *>(in + (t * rows + src) * (cols / 16) + 4 * c);
    *reinterpret_cast<uint32_t *>(out + atom * 512 + 16 * (r % 32) + 4 * (r / 32)) = word;
  }
}

// ------------------------------------------------------------------ padded slots
struct Tables {
  const int32_t *counts, *offsets, *active, *n_active, *tile_prefix, *perm;
};

// Padded slot p: the expert e and the rank j of the slot within e; false past the used
// range (the slot is then never read).  The slot holds a routed pair iff j < counts[e].
__device__ __forceinline__ bool pad_slot(const Tables &tb, int n_act, int64_t p, int &e, int &j) {
  if (n_act <= 0) return false;
  const int t = (int)(p / kPadN);
  if (t >= tb.tile_prefix[n_act]) return false;
  int lo = 0, hi = n_act - 1;
  while (lo < hi) {   // last a with tile_prefix[a] <= t
    const int mid = (lo + hi + 1) >> 1;
    if (tb.tile_prefix[mid] <= t)
      lo = mid;
    else
      hi = mid - 1;
  }
  e = tb.active[lo];
  j = (int)(p - (int64_t)tb.tile_prefix[lo] * kPadN);
  return true;
}

// One warp per padded slot: the activation row (MODE 0: the token's x row; MODE 1: the
// slot's h row) quantized as a tensor of its own, codes to q [P, cols/2], scales to atoms,
// the row's global scale to g[p] (0 for an empty slot, whose codes and scales are 0).
template <int MODE>
__global__ void __launch_bounds__(256) quant_rows_kernel(Tables tb, const __nv_bfloat16 *src,
                                                         int64_t cols, int64_t K, int64_t P,
                                                         uint8_t *__restrict__ q,
                                                         uint8_t *__restrict__ sf,
                                                         float *__restrict__ g_out) {
  pdl_wait();   // the routing tables (and h) come from the previous kernels
  const int n_act = *tb.n_active;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t nb = cols / 16;
  for (int64_t p = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; p < P; p += nwarps) {
    int e = 0, j = 0;
    if (!pad_slot(tb, n_act, p, e, j)) continue;
    const bool valid = j < tb.counts[e];
    const uint4 *row = nullptr;
    if (valid) {
      const int64_t slot = tb.offsets[e] + j;
      const int64_t r = MODE == 0 ? tb.perm[slot] / K : slot;
      row = reinterpret_cast<const uint4 *>(src + r * cols);
    }
    // the row's amax: integer max over the bf16 magnitudes (same order as the values)
    uint32_t m = 0;
    if (valid)
      for (int64_t i = lane; i < cols / 8; i += 32) {
        const uint4 v = __ldcg(row + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) m = max(m, max(w[k] & 0x7FFFu, (w[k] >> 16) & 0x7FFFu));
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const float g = global_scale_from_amax(m << 16);
    const BlockScaleConsts bc = block_scale_consts(g);
    if (lane == 0) g_out[p] = valid ? g : 0.f;
    uint2 *qrow = reinterpret_cast<uint2 *>(q + p * (cols / 2));
    for (int64_t b = lane; b < nb; b += 32) {
      uint2 codes = make_uint2(0u, 0u);
      uint32_t sc = 0;
      if (valid) codes = quantize_block16(__ldcg(row + 2 * b), __ldcg(row + 2 * b + 1), g, bc.c,
                                          bc.fast, &sc);
      qrow[b] = codes;
      sf[atom_offset(p, b, cols)] = (uint8_t)sc;
    }
  }
  pdl_launch_dependents();
}

// One warp per token: x quantized once per token (a token's slots all share its x row):
// codes [T, H/2], the scale bytes row-major [T, H/16], the global scale g[T].
__global__ void __launch_bounds__(256) quant_tokens_kernel(const __nv_bfloat16 *x, int64_t T,
                                                           int64_t H, uint8_t *__restrict__ q,
                                                           uint8_t *__restrict__ sc_rows,
                                                           float *__restrict__ g_out) {
  pdl_wait();   // x may come from the previous kernel
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
    const uint4 *row = reinterpret_cast<const uint4 *>(x + t * H);
    uint32_t m = 0;
    for (int64_t i = lane; i < H / 8; i += 32) {
      const uint4 v = __ldg(row + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) m = max(m, max(w[k] & 0x7FFFu, (w[k] >> 16) & 0x7FFFu));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const float g = global_scale_from_amax(m << 16);
    const BlockScaleConsts bc = block_scale_consts(g);
    if (lane == 0) g_out[t] = g;
    uint2 *qrow = reinterpret_cast<uint2 *>(q + t * (H / 2));
    for (int64_t b = lane; b < H / 16; b += 32) {
      uint32_t sc = 0;
      qrow[b] = quantize_block16(__ldg(row + 2 * b), __ldg(row + 2 * b + 1), g, bc.c, bc.fast, &sc);
      sc_rows[t * (H / 16) + b] = (uint8_t)sc;
    }
  }
  pdl_launch_dependents();
}

// One warp per padded slot: the slot's token's codes, scales (four blocks = one 32-bit word,
// the same word in both layouts) and global scale, copied into the slot; zeros for an empty
// slot.
__global__ void __launch_bounds__(256) gather_slots_kernel(Tables tb, int64_t H, int64_t K,
                                                           int64_t P, const uint8_t *q_tok,
                                                           const uint8_t *sc_tok,
                                                           const float *g_tok,
                                                           uint8_t *__restrict__ q,
                                                           uint8_t *__restrict__ sf,
                                                           float *__restrict__ g_out) {
  pdl_wait();   // routing tables and the token codes
  const int n_act = *tb.n_active;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t p = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; p < P; p += nwarps) {
    int e = 0, j = 0;
    if (!pad_slot(tb, n_act, p, e, j)) continue;
    const bool valid = j < tb.counts[e];
    const int64_t t = valid ? tb.perm[tb.offsets[e] + j] / K : 0;
    const uint4 *src = reinterpret_cast<const uint4 *>(q_tok + t * (H / 2));
    uint4 *dst = reinterpret_cast<uint4 *>(q + p * (H / 2));
    for (int64_t i = lane; i < H / 32; i += 32) dst[i] = valid ? __ldcg(src + i) : make_uint4(0, 0, 0, 0);
    const uint32_t *ssrc = reinterpret_cast<const uint32_t *>(sc_tok + t * (H / 16));
    for (int64_t c = lane; c < H / 64; c += 32)
      *reinterpret_cast<uint32_t *>(sf + atom_offset(p, 4 * c, H)) = valid ? __ldcg(ssrc + c) : 0u;
    if (lane == 0) g_out[p] = valid ? __ldcg(g_tok + t) : 0.f;
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ the block-scaled GEMM
constexpr int QS = 3;                            // pipeline stages (512 elements of K each)
constexpr uint32_t kQSub = 128 * 128;            // a 128-row tile 128 bytes (256 E2M1) wide
constexpr uint32_t kQA = 2 * kQSub;              // weight tile: 128 rows, two K halves
constexpr uint32_t kQB = 2 * kQSub;              // activation tile: 128 slots, two K halves
constexpr uint32_t kQSF = 8 * 512;               // eight scale atoms (512 elements of K)
constexpr uint32_t kQStage = kQA + kQB + 2 * kQSF;
// Epilogue scratch: the 16-slot chunk staged for coalesced stores (down: 16 x 132 fp32;
// gate/up: the exchanged gate and up halves, 2 x 64 x 9 fp32, then 16 x 64 bf16 of h), and
// the tile's per-slot factors (128 fp32).
constexpr uint32_t kQE = QS * kQStage;
constexpr uint32_t kQEBytes = 16 * 132 * 4;
constexpr uint32_t kQCol = kQE + kQEBytes;
constexpr uint32_t kQBars = kQCol + kPadN * 4;
constexpr uint32_t kQMisc = kQBars + 8 * (2 * QS + 4);
constexpr uint32_t kQSmem = kQMisc + 16 + 1024;  // + alignment slack
constexpr int kQThreads = 192;                   // producer, MMA, 4 epilogue warps
// TMEM: two accumulators of 128 columns, then two buffers each of 32 columns of weight
// scales and 32 of activation scales (eight atoms of four columns).
constexpr uint32_t kTmemSFA = 2 * kPadN, kTmemSFB = kTmemSFA + 64, kQTmemCols = 512;
static_assert(kQSmem <= 227 * 1024, "shared memory budget");
static_assert(kQStage % 1024 == 0 && kQSub % 1024 == 0, "swizzled tiles on 1024-byte boundaries");

struct W4Gemm {
  Tables tb;
  const float *w;            // [T*K] routing weights (down)
  const uint8_t *sfw;        // weight scale atoms
  const uint8_t *sfx;        // activation scale atoms
  const float *g_w;          // [E]
  const float *g_act;        // [P] per padded slot
  __nv_bfloat16 *h;          // gate/up output [T*K, I], slot order
  float *y;                  // down output [T*K, H], slot order
  int32_t *flag;
  int64_t H, I;
  int mode;                  // 0: gate/up + SwiGLU; 1: down
  int Kred;                  // reduction length (H or I), a multiple of 256
  int m_tiles, m_groups;     // 128-row tiles per expert; scale-atom row groups per expert
};

__global__ void __launch_bounds__(kQThreads, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                     const __grid_constant__ CUtensorMap tmap_x, W4Gemm p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kQBars);
  uint64_t *freeb = full + QS;
  uint64_t *accfull = freeb + QS;
  uint64_t *accempty = accfull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kQMisc);
  int *abort = reinterpret_cast<int *>(smem + kQMisc + 4);
  float *ebuf = reinterpret_cast<float *>(smem + kQE);
  float *colf = reinterpret_cast<float *>(smem + kQCol);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort = 0;
    for (int s = 0; s < QS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&freeb[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kQTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  pdl_wait();   // routing tables, quantized activations and their scales
  const int n_act = *p.tb.n_active;
  const int total = n_act > 0 ? p.tb.tile_prefix[n_act] * p.m_tiles : 0;
  const int kblocks = (p.Kred + 511) / 512;   // the last may hold one 256-element half
  const int64_t H = p.H, I = p.I;

  auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    if (*(volatile int *)abort) return false;
    if (mbar_wait(bar, parity)) return true;
    *(volatile int *)abort = 1;
    report_timeout(p.flag);
    return false;
  };
  // tile -> expert, rank of its n-tile within the expert, valid slots, first padded slot
  auto tile_of = [&](int tile, int &e, int &mt, int &nvalid, int64_t &pad0, int64_t &slot0) {
    const int t = tile / p.m_tiles;
    mt = tile % p.m_tiles;
    int j = 0;
    pad_slot(p.tb, n_act, (int64_t)t * kPadN, e, j);
    pad0 = (int64_t)t * kPadN;
    slot0 = p.tb.offsets[e] + j;
    nvalid = min(kPadN, p.tb.counts[e] - j);
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int kg = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        int e, mt, nvalid;
        int64_t pad0, slot0;
        tile_of(tile, e, mt, nvalid, pad0, slot0);
        const uint8_t *sfw = p.sfw + ((int64_t)e * p.m_groups + mt) * (p.Kred / 64) * 512;
        const uint8_t *sfx = p.sfx + (pad0 / kPadN) * (p.Kred / 64) * 512;
        for (int kb = 0; kb < kblocks; ++kb, ++kg) {
          const int s = kg % QS;
          if (kg >= QS && !wait(&freeb[s], ((kg / QS) - 1) & 1)) break;
          if (*(volatile int *)abort) break;
          const int nh = min(2, (p.Kred - kb * 512) / 256);   // K halves in this stage
          mbar_arrive_expect_tx(&full[s], (uint32_t)nh * (2 * kQSub + kQSF));
          unsigned char *A = smem + s * kQStage;
          for (int h = 0; h < nh; ++h) {
            const int x = kb * 256 + h * 128;   // byte column of the half
            unsigned char *Ah = A + h * kQSub;
            if (p.mode == 0) {   // 64 gate rows, then the matching 64 up rows
              tma_load_2d(Ah, &tmap_w, x, (int)(e * 2 * I + mt * 64), &full[s]);
              tma_load_2d(Ah + kQSub / 2, &tmap_w, x, (int)(e * 2 * I + I + mt * 64), &full[s]);
            } else {
              tma_load_2d(Ah, &tmap_w, x, (int)(e * H + mt * 128), &full[s]);
            }
            tma_load_2d(A + kQA + h * kQSub, &tmap_x, x, (int)pad0, &full[s]);
          }
          bulk_g2s(A + kQA + kQB, sfw + kb * kQSF, nh * (kQSF / 2), &full[s]);
          bulk_g2s(A + kQA + kQB + kQSF, sfx + kb * kQSF, nh * (kQSF / 2), &full[s]);
        }
        if (*(volatile int *)abort) break;
      }
      for (int t = max(0, kg - QS); t < kg; ++t) mbar_wait(&full[t % QS], (t / QS) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int kg = 0, tc = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tc) {
        int e, mt, nvalid;
        int64_t pad0, slot0;
        tile_of(tile, e, mt, nvalid, pad0, slot0);
        const int acc = tc & 1;
        if (tc >= 2 && !wait(&accempty[acc], ((tc >> 1) - 1) & 1)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kPadN;
        const uint32_t idesc = idesc_nvfp4_f32(128, max(16, (nvalid + 15) & ~15));
        for (int kb = 0; kb < kblocks; ++kb, ++kg) {
          const int s = kg % QS;
          const bool ok = wait(&full[s], (kg / QS) & 1);
          tc_fence_after();
          if (ok) {
            const int nk = 4 * min(2, (p.Kred - kb * 512) / 256);   // MMAs of K = 64
            const uint32_t st = smem_u32(smem + s * kQStage);
            const uint32_t sfa = tmem_base + kTmemSFA + 32 * (kg & 1);
            const uint32_t sfb = tmem_base + kTmemSFB + 32 * (kg & 1);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (i < nk) {
                tmem_cp_32x128b_x4(sfa + 4 * i, smem_desc_rows16(st + kQA + kQB + 512 * i));
                tmem_cp_32x128b_x4(sfb + 4 * i,
                                   smem_desc_rows16(st + kQA + kQB + kQSF + 512 * i));
              }
#pragma unroll
            for (int i = 0; i < 8; ++i)   // K = 64 E2M1 = 32 bytes along a 128-byte row
              if (i < nk) {
                const uint32_t half = (uint32_t)(i / 4) * kQSub;
                const uint64_t da = smem_desc_sw128(st + half);
                const uint64_t db = smem_desc_sw128(st + kQA + half);
                umma_nvfp4(d_tmem, da + 2 * (i % 4), db + 2 * (i % 4), idesc, sfa + 4 * i,
                           sfb + 4 * i, kb > 0 || i > 0);
              }
          }
          umma_commit(&freeb[s]);
        }
        umma_commit(&accfull[acc]);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2-5)
    // Warp w reads TMEM lanes 32 (w % 4) .. +31: lane L is weight row L of the tile.  A chunk
    // of 16 slots leaves through shared memory, so every global store is a 16-byte piece of
    // one slot's row.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 64;   // 0..127
    int tc = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tc) {
      int e, mt, nvalid;
      int64_t pad0, slot0;
      tile_of(tile, e, mt, nvalid, pad0, slot0);
      const int acc = tc & 1;
      if (!wait(&accfull[acc], (tc >> 1) & 1)) break;
      tc_fence_after();
      {   // the slot's factor: g_w * g_row, times the routing weight for down
        float f = 0.f;
        if (et < nvalid) {
          f = __ldg(p.g_w + e) * __ldg(p.g_act + pad0 + et);
          if (p.mode == 1) f *= __ldg(p.w + __ldg(p.tb.perm + slot0 + et));
        }
        colf[et] = f;
      }
      named_sync(1, 128);
      const uint32_t tbase = tmem_base + acc * kPadN + ((uint32_t)(q * 32) << 16);
      for (int c0 = 0; c0 < nvalid; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tbase + c0, v);
        float val[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) val[c] = __uint_as_float(v[c]) * colf[c0 + c];
        if (p.mode == 0) {
          // gate rows (lanes 0-63) keep columns 0-7 and hand over 8-15; up rows the reverse
          float *G = ebuf, *U = ebuf + 64 * 9;
          __nv_bfloat16 *hs = reinterpret_cast<__nv_bfloat16 *>(ebuf + 128 * 9);   // [16][64]
          if (q < 2) {
#pragma unroll
            for (int c = 0; c < 8; ++c) G[row * 9 + c] = val[8 + c];
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) U[(row - 64) * 9 + c] = val[c];
          }
          named_sync(1, 128);
          if (q < 2) {
#pragma unroll
            for (int c = 0; c < 8; ++c)
              hs[c * 64 + row] = __float2bfloat16_rn(silu_fast(val[c]) * U[row * 9 + c]);
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c)
              hs[(8 + c) * 64 + row - 64] =
                  __float2bfloat16_rn(silu_fast(G[(row - 64) * 9 + c]) * val[8 + c]);
          }
          named_sync(1, 128);
          const int c = et >> 3, part = et & 7;   // 16 slots x 8 pieces of 16 bytes
          if (c0 + c < nvalid)
            *reinterpret_cast<uint4 *>(p.h + (slot0 + c0 + c) * I + mt * 64 + part * 8) =
                *reinterpret_cast<const uint4 *>(hs + c * 64 + part * 8);
          named_sync(1, 128);
        } else {
          float *ys = ebuf;   // [16][132]
#pragma unroll
          for (int c = 0; c < 16; ++c) ys[c * 132 + row] = val[c];
          named_sync(1, 128);
#pragma unroll
          for (int k = 0; k < 4; ++k) {   // 16 slots x 32 pieces of 16 bytes
            const int pi = et + 128 * k, c = pi >> 5, part = pi & 31;
            if (c0 + c < nvalid)
              *reinterpret_cast<float4 *>(p.y + (slot0 + c0 + c) * H + mt * 128 + part * 4) =
                  *reinterpret_cast<const float4 *>(ys + c * 132 + part * 4);
          }
          named_sync(1, 128);
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
    tmem_dealloc(tmem_base, kQTmemCols);
  }
}

// Workspace of the W4A4 forward: the routed forward's, then the quantized activations.
struct W4Layout {
  size_t base, xq, xsf, gx, hq, hsf, gh, xq_tok, xsc_tok, gx_tok, total;
  int64_t P;   // padded slots provided for
};
W4Layout w4a4_layout(int64_t T, int64_t H, int64_t I, int64_t E, int64_t K) {
  W4Layout L = {};
  L.base = workspace_layout(T, H, I, E, K).total;
  L.P = round_up(T * K + std::min<int64_t>(E, T * K) * (kPadN - 1), kPadN);
  size_t o = L.base;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += (bytes + 1023) & ~size_t(1023);
    return at;
  };
  L.xq = take((size_t)(L.P * H / 2));
  L.xsf = take((size_t)(L.P * H / 16));
  L.gx = take((size_t)(L.P * 4));
  L.hq = take((size_t)(L.P * I / 2));
  L.hsf = take((size_t)(L.P * I / 16));
  L.gh = take((size_t)(L.P * 4));
  L.xq_tok = take((size_t)(T * H / 2));
  L.xsc_tok = take((size_t)(T * H / 16));
  L.gx_tok = take((size_t)(T * 4));
  L.total = o;
  return L;
}

int launch_quant_rows(int mode, const Tables &tb, const __nv_bfloat16 *src, int64_t cols,
                      int64_t K, int64_t P, uint8_t *q, uint8_t *sf, float *g, cudaStream_t s) {
  const int64_t blocks = std::min<int64_t>(ceil_div(P * 32, 256), (int64_t)num_sms() * 8);
  return mode == 0
             ? launch_pdl(quant_rows_kernel<0>, dim3((unsigned)blocks), dim3(256), 0, s, tb, src,
                          cols, K, P, q, sf, g)
             : launch_pdl(quant_rows_kernel<1>, dim3((unsigned)blocks), dim3(256), 0, s, tb, src,
                          cols, K, P, q, sf, g);
}

int launch_w4a4_gemm(const W4Gemm &p, const uint8_t *wq, int64_t w_rows, const uint8_t *xq,
                     int64_t P, cudaStream_t s) {
  CUtensorMap tw, tx;
  // packed weights [E * rows, Kred/2] bytes: boxes of 64 (gate/up) or 128 (down) rows x 128 B
  if (make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, wq, (uint64_t)(p.Kred / 2),
               (uint64_t)w_rows, 128, p.mode == 0 ? 64 : 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return NVFP4_ECUDA;
  // quantized activations [P, Kred/2] bytes: boxes of 128 slots x 128 B
  if (make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, xq, (uint64_t)(p.Kred / 2), (uint64_t)P,
               128, kPadN, CU_TENSOR_MAP_SWIZZLE_128B))
    return NVFP4_ECUDA;
  if (resident_blocks(w4a4_gemm_kernel, kQThreads, kQSmem) <= 0) return NVFP4_ECUDA;
  return launch_pdl(w4a4_gemm_kernel, dim3(num_sms()), dim3(kQThreads), kQSmem, s, tw, tx, p);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// A timing mark between two kernels (external event under stream capture).
int mark(cudaEvent_t const *ev, int i, cudaStream_t s) {
  if (!ev) return NVFP4_OK;
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &st);
  if (e == cudaSuccess)
    e = st == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev[i], s, cudaEventRecordExternal)
                                            : cudaEventRecord(ev[i], s);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  return NVFP4_OK;
}

}  // namespace

// The W4A4 forward, with timing marks between the stages when ev is not null.
int forward_w4a4(const __nv_bfloat16 *x, const int32_t *topk_ids, const float *topk_w, int64_t T,
                 int64_t H, int64_t I, int64_t E, int64_t K, const uint8_t *w_gu,
                 const uint8_t *sf_gu, const float *g_gu, const uint8_t *w_dn,
                 const uint8_t *sf_dn, const float *g_dn, __nv_bfloat16 *out, void *workspace,
                 size_t ws_bytes, cudaEvent_t const *ev, cudaStream_t stream);
}  // namespace nvfp4

using namespace nvfp4;

extern "C" int nvfp4_w4a4_prepare_scales(const uint8_t *scales, int64_t n_tensors, int64_t rows,
                                         int64_t cols, int64_t gate_rows, uint8_t *out,
                                         cudaStream_t stream) {
  if (!scales || !out || n_tensors <= 0 || rows <= 0 || cols <= 0 || gate_rows < 0)
    return NVFP4_EINVAL;
  if (cols % 64 || rows % 128 || (gate_rows && (gate_rows % 64 || 2 * gate_rows != rows)))
    return NVFP4_ESHAPE;
  if ((reinterpret_cast<uintptr_t>(scales) | reinterpret_cast<uintptr_t>(out)) & 3)
    return NVFP4_EINVAL;
  const int64_t total = n_tensors * (rows / 128) * (cols / 64) * 128;
  const int64_t blocks = std::min<int64_t>(ceil_div(total, 256), (int64_t)num_sms() * 16);
  swizzle_scales_kernel<<<(unsigned)blocks, 256, 0, stream>>>(scales, n_tensors, rows, cols,
                                                              gate_rows, out);
  return check_launch();
}

extern "C" size_t moe_nvfp4_w4a4_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E,
                                                int64_t K) {
  if (T <= 0 || H <= 0 || I <= 0 || E <= 0 || K <= 0) return 0;
  return w4a4_layout(T, H, I, E, K).total;
}

extern "C" int moe_nvfp4_forward_w4a4(const __nv_bfloat16 *x, const int32_t *topk_ids,
                                      const float *topk_w, int64_t T, int64_t H, int64_t I,
                                      int64_t E, int64_t K, const uint8_t *w_gu,
                                      const uint8_t *sf_gu, const float *g_gu,
                                      const uint8_t *w_dn, const uint8_t *sf_dn,
                                      const float *g_dn, __nv_bfloat16 *out, void *workspace,
                                      size_t ws_bytes, cudaStream_t stream) {
  return forward_w4a4(x, topk_ids, topk_w, T, H, I, E, K, w_gu, sf_gu, g_gu, w_dn, sf_dn, g_dn,
                      out, workspace, ws_bytes, nullptr, stream);
}

extern "C" int moe_nvfp4_forward_w4a4_profiled(
    const __nv_bfloat16 *x, const int32_t *topk_ids, const float *topk_w, int64_t T, int64_t H,
    int64_t I, int64_t E, int64_t K, const uint8_t *w_gu, const uint8_t *sf_gu, const float *g_gu,
    const uint8_t *w_dn, const uint8_t *sf_dn, const float *g_dn, __nv_bfloat16 *out,
    void *workspace, size_t ws_bytes, void *const *stage_events, cudaStream_t stream) {
  if (!stage_events) return NVFP4_EINVAL;
  for (int i = 0; i < 5; ++i)
    if (!stage_events[i]) return NVFP4_EINVAL;
  return forward_w4a4(x, topk_ids, topk_w, T, H, I, E, K, w_gu, sf_gu, g_gu, w_dn, sf_dn, g_dn,
                      out, workspace, ws_bytes,
                      reinterpret_cast<cudaEvent_t const *>(stage_events), stream);
}

int nvfp4::forward_w4a4(const __nv_bfloat16 *x, const int32_t *topk_ids, const float *topk_w,
                        int64_t T, int64_t H, int64_t I, int64_t E, int64_t K,
                        const uint8_t *w_gu, const uint8_t *sf_gu, const float *g_gu,
                        const uint8_t *w_dn, const uint8_t *sf_dn, const float *g_dn,
                        __nv_bfloat16 *out, void *workspace, size_t ws_bytes,
                        cudaEvent_t const *ev, cudaStream_t stream) {
  if (!x || !topk_ids || !topk_w || !w_gu || !sf_gu || !g_gu || !w_dn || !sf_dn || !g_dn || !out)
    return NVFP4_EINVAL;
  if (T <= 0 || H <= 0 || I <= 0 || E <= 0 || K <= 0) return NVFP4_EINVAL;
  if (H % 256 || I % 256 || K > 16 || E > kMaxExperts || T * K >= (int64_t(1) << 31) ||
      E * 2 * I >= (int64_t(1) << 31) || E * H >= (int64_t(1) << 31))
    return NVFP4_ESHAPE;
  if (!aligned16(x) || !aligned16(w_gu) || !aligned16(w_dn) || !aligned16(out) ||
      !aligned16(sf_gu) || !aligned16(sf_dn))
    return NVFP4_EINVAL;
  const W4Layout W = w4a4_layout(T, H, I, E, K);
  if (!workspace || !aligned16(workspace) || ws_bytes < W.total) return NVFP4_EWORKSPACE;
  if (W.P >= (int64_t(1) << 31)) return NVFP4_ESHAPE;
  const WorkspaceLayout L = workspace_layout(T, H, I, E, K);
  char *ws = static_cast<char *>(workspace);

  MoeArgs a = {};
  a.x = x;
  a.ids = topk_ids;
  a.w = topk_w;
  a.out = out;
  a.T = T;
  a.H = H;
  a.I = I;
  a.E = E;
  a.K = K;
  a.map = whole_layer(E);
  a.flag = reinterpret_cast<int32_t *>(ws + L.flag);
  a.n_active = reinterpret_cast<int32_t *>(ws + L.n_active);
  a.counts = reinterpret_cast<int32_t *>(ws + L.counts);
  a.offsets = reinterpret_cast<int32_t *>(ws + L.offsets);
  a.active = reinterpret_cast<int32_t *>(ws + L.active);
  a.tile_prefix = reinterpret_cast<int32_t *>(ws + L.tile_prefix);
  a.perm = reinterpret_cast<int32_t *>(ws + L.perm);
  a.inv = reinterpret_cast<int32_t *>(ws + L.inv);
  a.h = reinterpret_cast<__nv_bfloat16 *>(ws + L.h);
  a.y = reinterpret_cast<float *>(ws + L.y);

  RouteArgs r = {};
  r.ids = topk_ids;
  r.n_pairs = T * K;
  r.E = (int)E;
  r.map = a.map;
  r.counts = a.counts;
  r.offsets = a.offsets;
  r.perm = a.perm;
  r.inv = a.inv;
  r.flag = a.flag;
  r.active = a.active;
  r.n_active = a.n_active;
  r.tile_prefix = a.tile_prefix;
  r.tile_n = kPadN;
  if (int s = mark(ev, 0, stream)) return s;
  if (int s = launch_route(r, stream, true, reinterpret_cast<int32_t *>(ws + L.route_blk)))
    return s;

  const Tables tb = {a.counts, a.offsets, a.active, a.n_active, a.tile_prefix, a.perm};
  uint8_t *xq = reinterpret_cast<uint8_t *>(ws + W.xq), *xsf = reinterpret_cast<uint8_t *>(ws + W.xsf);
  uint8_t *hq = reinterpret_cast<uint8_t *>(ws + W.hq), *hsf = reinterpret_cast<uint8_t *>(ws + W.hsf);
  float *gx = reinterpret_cast<float *>(ws + W.gx), *gh = reinterpret_cast<float *>(ws + W.gh);
  {   // x: each token quantized once, then copied into its slots
    uint8_t *q_tok = reinterpret_cast<uint8_t *>(ws + W.xq_tok);
    uint8_t *s_tok = reinterpret_cast<uint8_t *>(ws + W.xsc_tok);
    float *g_tok = reinterpret_cast<float *>(ws + W.gx_tok);
    const int64_t bt = std::min<int64_t>(ceil_div(T * 32, 256), (int64_t)num_sms() * 8);
    if (int s = launch_pdl(quant_tokens_kernel, dim3((unsigned)bt), dim3(256), 0, stream, x, T,
                           H, q_tok, s_tok, g_tok))
      return s;
    const int64_t bp = std::min<int64_t>(ceil_div(W.P * 32, 256), (int64_t)num_sms() * 8);
    if (int s = launch_pdl(gather_slots_kernel, dim3((unsigned)bp), dim3(256), 0, stream, tb, H,
                           K, W.P, (const uint8_t *)q_tok, (const uint8_t *)s_tok,
                           (const float *)g_tok, xq, xsf, gx))
      return s;
  }
  if (int s = mark(ev, 1, stream)) return s;

  W4Gemm g = {};
  g.tb = tb;
  g.w = topk_w;
  g.flag = a.flag;
  g.H = H;
  g.I = I;
  g.mode = 0;
  g.Kred = (int)H;
  g.m_tiles = (int)(I / 64);
  g.m_groups = (int)(2 * I / 128);
  g.sfw = sf_gu;
  g.sfx = xsf;
  g.g_w = g_gu;
  g.g_act = gx;
  g.h = a.h;
  if (int s = launch_w4a4_gemm(g, w_gu, E * 2 * I, xq, W.P, stream)) return s;
  if (int s = mark(ev, 2, stream)) return s;

  if (int s = launch_quant_rows(1, tb, a.h, I, K, W.P, hq, hsf, gh, stream)) return s;

  g.mode = 1;
  g.Kred = (int)I;
  g.m_tiles = (int)(H / 128);
  g.m_groups = (int)(H / 128);
  g.sfw = sf_dn;
  g.sfx = hsf;
  g.g_w = g_dn;
  g.g_act = gh;
  g.y = a.y;
  if (int s = launch_w4a4_gemm(g, w_dn, E * H, hq, W.P, stream)) return s;
  if (int s = mark(ev, 3, stream)) return s;
  if (int s = launch_combine(a, stream)) return s;
  return mark(ev, 4, stream);
}
