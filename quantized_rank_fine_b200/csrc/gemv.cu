// Small-M forward: Y = X deq(Wq) + V B for M <= 16 tokens (NF4 dequant-GEMV).
//
// At a few tokens the forward is bound by reading the 4-bit codes once from HBM
// (0.516 B per weight), so the kernel is organised around that stream:
//
//   * Work unit: a 256-column tile of W (four absmax blocks, 128 contiguous bytes
//     of codes per row) times a K-range.  Whole 128-byte lines per row keep the
//     HBM reads dense; the tiles running side by side cover whole rows at once.
//     The grid (tiles x K-splits) is sized to be resident at once, two CTAs per
//     SM.  A producer warp streams, with TMA, 64 rows of the tile's codes (8 KB,
//     128-byte swizzle) and the matching 64 columns of X per stage through a
//     6-stage shared-memory ring.  Consumer warp w takes column group w & 3 (one
//     absmax block, 64 columns) and row half w >> 2 of every stage.
//   * Tensor cores, swap-AB: mma.sync m16n8k16 with the weight as the 16 x 16 A
//     operand (rows = 16 output columns, cols = 16 k) and the tokens as the 8-wide
//     B operand.  Lane (g, t) reads one 32-bit word (8 codes, output columns
//     8g .. 8g+7 of its group) from rows 2t, 2t+1, 2t+8, 2t+9 of a 16-row step;
//     with the swizzle the 32 lanes hit 32 banks.  Two bit-selects re-pair the
//     nibbles so that byte j of a word holds the codes of two consecutive rows
//     (k, k+1) of one column; a 256-entry shared table (32 copies, one per lane:
//     no bank conflicts) maps that byte to the bf16 pair (level(k), level(k+1)),
//     which is exactly one A register.
//   * The block scale is folded into the activations: sum_k x_k (a'_k l_k) =
//     sum_k (x_k a'_k) l_k.  The B fragment is x'[m][k] = bf16(x[m][k] * a'(k, block)),
//     built in registers from the X tile and the block's absmax'; the weight
//     operand is the bf16 NF4 level itself.  Each lane computes a' of one row of
//     its warp's block per stage from an absmax code and scale it loaded two
//     stages earlier, so nothing runs before the first stage but the level table.
//   * A consumer warp takes the weight stages two at a time: it waits for both,
//     then runs their four 16-row steps as one stretch of code, so the table
//     lookups and products of the two stages overlap.
//   * The adapter term V B rides on the same MMAs as r extra k rows of the last
//     K-split, [X | V] [deq(Wq); B]: its producer loads, per 16 adapter rows, the
//     tile's 16 x 256 block of B (TMA, 128-byte swizzle) and the 16 matching
//     columns of V into a ring stage; the A registers pair two B rows of one
//     column with a byte-permute and the B fragment is V itself.
//   * V comes from the kernel launched just before (X A).  Launched as a
//     programmatic dependent, this kernel streams all of its codes while that
//     one finishes; only the last split's producer waits for it, before it loads V.
//     It lets its own dependent (the next call's first kernel, which waits for
//     this one to finish before it reads anything) become resident at once.
//   * The K-splits of a tile form one thread-block cluster; the split count
//     follows from how many clusters of each size the device holds at once (see
//     gemv_plan: the fewest waves x rows per CTA at up to 8 tokens, the fewest
//     stages per SM above).  Each CTA sums its row halves into
//     an fp32 [M][256] partial and stores each slice of it straight into the
//     shared memory of the CTA that owns the slice (distributed shared memory);
//     after one cluster barrier every owner adds its slices in split order
//     (the result does not depend on timing) and writes bf16 Y.  No global
//     scratch, no atomics, no remote loads.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

namespace qlora {

namespace {

using namespace sm100;

constexpr int kGvConsumers = 8;                       // 4 column groups x 2 row halves
constexpr int kGvThreads = (kGvConsumers + 1) * 32;   // + 1 producer warp
constexpr int kTileCols = 256;
constexpr int kStageRows = 64;
constexpr int kGvStages = 6;
constexpr uint32_t kCodeBytes = kStageRows * 128;     // 64 rows x 128 bytes
constexpr uint32_t kXBytes = 16 * 128;                // 64 columns of X for up to 16 tokens
constexpr uint32_t kStageBytes = kCodeBytes + kXBytes;   // a multiple of 1024 (swizzle atoms)
constexpr int kLutCopies = 32;
constexpr int kLutBytes = 256 * kLutCopies * 4;       // 32 copies of the 256-entry table
constexpr int kMaxCluster = 16;                       // K-splits per tile
// receive buffer of the split-K reduction: <= 16 x 64 groups of 4 floats plus
// the rounding of one group per owner
constexpr int kRecvBytes = (16 * 64 + kMaxCluster) * 16;

static_assert(kStageBytes % 1024 == 0, "stage buffers must stay 1024-byte aligned");

struct GemvArgs {
  const uint8_t* dq_codes;
  const float* dq_scales;
  int64_t K, N;          // weight (K = in, N = out)
  int M;                 // tokens, 1..16
  int r;                 // adapter rank (V is M x r, B is r x N, bf16)
  uint16_t* Y;           // (M, N) bf16
  int Kc;                // rows per split (multiple of 64)
  uint32_t* status;
  int dq_u8;             // absmax codes are linear uint8 (else E4M3)
};

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Level pair of byte J of `x` from this lane's copy of the shared level table
// (entries 128 bytes apart, copy = lane): prmt extracts the byte and one
// multiply-add forms the address.  `k128` is 128 passed at run time so that the
// multiply stays an integer multiply-add (FMA pipe) instead of becoming a shift
// on the integer ALU pipe, which the extraction already loads.
template <int J>
__device__ __forceinline__ uint32_t lut_pair(uint32_t lut_lane, uint32_t x, uint32_t k128) {
  uint32_t v;
  asm("{\n\t.reg .b32 b, a;\n\t"
      "prmt.b32 b, %1, 0, %4;\n\t"
      "mad.lo.u32 a, b, %3, %2;\n\t"
      "ld.shared.b32 %0, [a];\n\t}"
      : "=r"(v)
      : "r"(x), "r"(lut_lane), "r"(k128), "n"(0x4440 | J));
  return v;
}

// 32-bit word at byte `byte` (a multiple of 4) of row `row` of a 1024-byte-aligned
// tile of 128-byte rows written by TMA with the 128-byte swizzle (the 16-byte
// chunk index is XORed with the row index mod 8).
__device__ __forceinline__ uint32_t ld_sw128(const uint8_t* tile, int row, int byte) {
  return *reinterpret_cast<const uint32_t*>(tile + row * 128 + ((((byte >> 4) ^ row) & 7) << 4) + (byte & 15));
}

template <int MT>   // token tiles of 8: 1 (M <= 8) or 2 (M <= 16)
__global__ void __launch_bounds__(kGvThreads, 2)
nf4_gemv_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_v,
                const GemvArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;                                                  // kGvStages x (codes, X)
  uint8_t* lut = smem + kGvStages * kStageBytes;                         // [256][32] x 4 bytes
  float* aslice = reinterpret_cast<float*>(lut + kLutBytes);             // [8 warps][2][32] absmax'
  float* part = reinterpret_cast<float*>(ring);                          // [M][256] after the loop
  float* recv = aslice + kGvConsumers * 64;                              // [S][cap] float4
  __shared__ __align__(8) uint64_t bars[2 * kGvStages];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  grid_launch_dependents();
  const int tile = blockIdx.x, split = blockIdx.y;
  const int64_t k_begin = static_cast<int64_t>(split) * p.Kc;
  const int rows = static_cast<int>(p.K - k_begin < p.Kc ? p.K - k_begin : p.Kc);   // multiple of 64
  const int nstage = rows / kStageRows;
  // the last split also takes the adapter rows, 16 per stage
  const int nall = nstage + (split == static_cast<int>(gridDim.y) - 1 ? (p.r + 15) / 16 : 0);
  const int64_t col0 = static_cast<int64_t>(tile) * kTileCols;
  const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + kGvStages);

  if (tid == 0) {
    for (int s = 0; s < kGvStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kGvConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();

  float acc[MT][4][4];
#pragma unroll
  for (int a = 0; a < MT; ++a)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][j][c] = 0.0f;

  const int cg = warp & 3, half = warp >> 2;
  if (warp == kGvConsumers) {
    // ------------------------------------------------------------ producer (one lane)
    if (lane == 0) {
      const uint32_t x_bytes = static_cast<uint32_t>(p.M) * 128;
      const uint32_t v_bytes = static_cast<uint32_t>(p.M) * 32;
      tma_prefetch_desc(&tm_codes);
      tma_prefetch_desc(&tm_x);
      int issued = 0;
      for (int i = 0; i < nall; ++i) {
        const int s = i % kGvStages;
        const uint32_t ph = (i / kGvStages) & 1;
        if (i >= kGvStages && !mbar_wait(empty0 + 8 * s, ph ^ 1, p.status, kFlagTimeoutProducer)) break;
        const uint32_t dst = smem_addr(ring + s * kStageBytes);
        if (i < nstage) {
          const int32_t k = static_cast<int32_t>(k_begin + i * kStageRows);
          mbar_arrive_expect_tx(full0 + 8 * s, kCodeBytes + x_bytes);
          tma_load_2d(dst, &tm_codes, full0 + 8 * s, tile * 128, k);
          tma_load_2d(dst + kCodeBytes, &tm_x, full0 + 8 * s, k, 0);
        } else {
          if (i == nstage) grid_dependency_wait();   // V is written by the preceding kernel
          const int32_t j0 = (i - nstage) * 16;
          mbar_arrive_expect_tx(full0 + 8 * s, 4 * 2048 + v_bytes);
          for (int c = 0; c < 4; ++c)
            tma_load_2d(dst + c * 2048, &tm_b, full0 + 8 * s, tile * kTileCols + 64 * c, j0);
          tma_load_2d(dst + kCodeBytes, &tm_v, full0 + 8 * s, j0, 0);
        }
        issued = i + 1;
      }
      // The ring becomes the partial buffer below: make sure none of the copies
      // issued last is still in flight (immediate unless a consumer gave up).
      for (int i = issued > kGvStages ? issued - kGvStages : 0; i < issued; ++i)
        mbar_wait(full0 + 8 * (i % kGvStages), (i / kGvStages) & 1, p.status, kFlagTimeoutProducer);
    }
  } else {
    // ------------------------------------------------------------ consumers
    // Level pairs of every byte, 32 copies (copy c serves lane c): entry e =
    // (level(e & 15), level(e >> 4)); each warp stores 512 contiguous bytes.
    {
      uint4* dst = reinterpret_cast<uint4*>(lut);
#pragma unroll
      for (int u = 0; u < kLutBytes / 16 / (kGvConsumers * 32); ++u) {
        const int q = tid + u * kGvConsumers * 32;   // uint4 index; 8 per entry
        const int e = q >> 3;
        const uint32_t v = pack_bf16x2(c_nf4_level[e & 15], c_nf4_level[e >> 4]);
        dst[q] = make_uint4(v, v, v, v);
      }
    }
    // absmax' of row (half*32 + lane) of each stage, block cg, from an absmax
    // code and scale loaded two stages ahead (zero past the last block of a row)
    const int64_t blocks_per_row = p.N / kBlock;
    const int64_t blk = static_cast<int64_t>(tile) * 4 + cg;
    const bool blk_ok = blk < blocks_per_row;
    auto load_scale = [&](int i, uint32_t& qc, float& qs) {
      qc = 0u;
      qs = 0.0f;
      if (blk_ok && i < nstage) {
        const int64_t b = (k_begin + i * kStageRows + half * 32 + lane) * blocks_per_row + blk;
        qc = __ldg(p.dq_codes + b);
        qs = __ldg(p.dq_scales + b / kGroup);
      }
    };
    const uint32_t lut_lane = smem_addr(lut) + lane * 4;
    float* asl = aslice + warp * 64;   // two slices: the stages of a pair
    constexpr uint32_t kLo = 0x0F0F0F0Fu;
    // 16, 2^28 and 128 as run-time values (p.M < 2^16): multiplies by them stay
    // multiply-adds on the FMA pipe rather than shifts on the integer pipe
    const uint32_t k16 = 16u | (static_cast<uint32_t>(p.M) >> 16);
    const uint32_t k2p28 = (1u << 28) | (static_cast<uint32_t>(p.M) >> 16);
    const uint32_t k128 = 128u | (static_cast<uint32_t>(p.M) >> 16);

    // One 16-row step (h = 0, 1 of this warp's row half) of the weight stage at
    // ctile, with the absmax' slice asl_s of that stage.
    auto hstep = [&](const uint8_t* ctile, const float* asl_s, int h) {
      const uint8_t* xtile = ctile + kCodeBytes;
      const int r0 = half * 32 + h * 16;   // first row of the 16-row step within the stage
      const int kb = cg * 32 + 4 * g;      // byte of this lane's 8 columns within the row
      const uint32_t c0 = ld_sw128(ctile, r0 + 2 * t, kb);
      const uint32_t c1 = ld_sw128(ctile, r0 + 2 * t + 1, kb);
      const uint32_t c2 = ld_sw128(ctile, r0 + 2 * t + 8, kb);
      const uint32_t c3 = ld_sw128(ctile, r0 + 2 * t + 9, kb);
      // byte j: (row k code, row k+1 code) of column 8g+2j (even) or 8g+2j+1 (odd);
      // c * 16 = c << 4 and umulhi(c, 2^28) = c >> 4
      const uint32_t e01 = (c0 & kLo) | ((c1 * k16) & ~kLo);
      const uint32_t o01 = (__umulhi(c0, k2p28) & kLo) | (c1 & ~kLo);
      const uint32_t e89 = (c2 & kLo) | ((c3 * k16) & ~kLo);
      const uint32_t o89 = (__umulhi(c2, k2p28) & kLo) | (c3 & ~kLo);
      // x' fragment: token a*8+g, k slots (2t, 2t+1) and (2t+8, 2t+9)
      const float2 s01 = *reinterpret_cast<const float2*>(asl_s + h * 16 + 2 * t);
      const float2 s89 = *reinterpret_cast<const float2*>(asl_s + h * 16 + 2 * t + 8);
      uint32_t bx[MT][2];
#pragma unroll
      for (int a = 0; a < MT; ++a) {
        const int m = a * 8 + g;
        bx[a][0] = 0u;
        bx[a][1] = 0u;
        if (m < p.M) {
          const uint32_t x01 = ld_sw128(xtile, m, 2 * (r0 + 2 * t));
          const uint32_t x89 = ld_sw128(xtile, m, 2 * (r0 + 2 * t + 8));
          bx[a][0] = pack_bf16x2(mul_rn(bf16_lo(x01), s01.x), mul_rn(bf16_hi(x01), s01.y));
          bx[a][1] = pack_bf16x2(mul_rn(bf16_lo(x89), s89.x), mul_rn(bf16_hi(x89), s89.y));
        }
      }
      auto tile_j = [&](auto jc) {
        constexpr int j = decltype(jc)::value;
        const uint32_t a0 = lut_pair<j>(lut_lane, e01, k128), a1 = lut_pair<j>(lut_lane, o01, k128);
        const uint32_t a2 = lut_pair<j>(lut_lane, e89, k128), a3 = lut_pair<j>(lut_lane, o89, k128);
#pragma unroll
        for (int a = 0; a < MT; ++a) mma_bf16_16816(acc[a][j], a0, a1, a2, a3, bx[a][0], bx[a][1]);
      };
      tile_j(std::integral_constant<int, 0>{});
      tile_j(std::integral_constant<int, 1>{});
      tile_j(std::integral_constant<int, 2>{});
      tile_j(std::integral_constant<int, 3>{});
    };

    // One stage; (qc, qs) hold its absmax code and scale and are reloaded with
    // those of stage i + 2 once used.  False if the wait for the stage timed out.
    auto stage = [&](int i, uint32_t& qc, float& qs) -> bool {
      const int s = i % kGvStages;
      const uint32_t ph = (i / kGvStages) & 1;
      if (i < nstage) {
        asl[lane] = absmax_deq(static_cast<uint8_t>(qc), qs, p.dq_u8 != 0);
        load_scale(i + 2, qc, qs);
        __syncwarp();   // the slice is complete
      }
      const bool got = mbar_wait(full0 + 8 * s, ph, p.status, kFlagTimeoutMma);
      if (!__all_sync(0xffffffffu, got)) return false;
      const uint8_t* ctile = ring + s * kStageBytes;
      const uint8_t* xtile = ctile + kCodeBytes;
      if (i >= nstage) {
        // adapter rows j0 .. j0+15: A = (B[j][col], B[j+1][col]), B fragment = V
        if (half == 0) {
          const uint8_t* btile = ctile + cg * 2048;   // [16 rows][64 columns] bf16, swizzled
          uint32_t bv[MT][2];
#pragma unroll
          for (int a = 0; a < MT; ++a) {
            const int m = a * 8 + g;
            bv[a][0] = m < p.M ? *reinterpret_cast<const uint32_t*>(xtile + m * 32 + 4 * t) : 0u;
            bv[a][1] = m < p.M ? *reinterpret_cast<const uint32_t*>(xtile + m * 32 + 16 + 4 * t) : 0u;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int cb = 2 * (8 * g + 2 * j);   // byte of columns (8g+2j, 8g+2j+1) in a row
            const uint32_t w0 = ld_sw128(btile, 2 * t, cb), w1 = ld_sw128(btile, 2 * t + 1, cb);
            const uint32_t w8 = ld_sw128(btile, 2 * t + 8, cb), w9 = ld_sw128(btile, 2 * t + 9, cb);
            const uint32_t a0 = __byte_perm(w0, w1, 0x5410), a1 = __byte_perm(w0, w1, 0x7632);
            const uint32_t a2 = __byte_perm(w8, w9, 0x5410), a3 = __byte_perm(w8, w9, 0x7632);
#pragma unroll
            for (int a = 0; a < MT; ++a) mma_bf16_16816(acc[a][j], a0, a1, a2, a3, bv[a][0], bv[a][1]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
        return true;
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) hstep(ctile, asl, h);
      __syncwarp();   // every lane is done with this stage and with the absmax' slice
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
      return true;
    };
    // Two weight stages at once: both waits first, then the four 16-row steps in
    // one stretch of code, so that the table lookups and products of both stages
    // overlap.  (qa, sa) and (qb, sb) hold the absmax data of stages i and i + 1.
    uint32_t qa, qb;
    float sa, sb;
    auto stage2 = [&](int i) -> bool {
      const int s0 = i % kGvStages, s1 = (i + 1) % kGvStages;
      asl[lane] = absmax_deq(static_cast<uint8_t>(qa), sa, p.dq_u8 != 0);
      asl[32 + lane] = absmax_deq(static_cast<uint8_t>(qb), sb, p.dq_u8 != 0);
      load_scale(i + 2, qa, sa);
      load_scale(i + 3, qb, sb);
      __syncwarp();   // both slices are complete
      const bool got = mbar_wait(full0 + 8 * s0, (i / kGvStages) & 1, p.status, kFlagTimeoutMma) &&
                       mbar_wait(full0 + 8 * s1, ((i + 1) / kGvStages) & 1, p.status, kFlagTimeoutMma);
      if (!__all_sync(0xffffffffu, got)) return false;
      const uint8_t* t0 = ring + s0 * kStageBytes;
      const uint8_t* t1 = ring + s1 * kStageBytes;
      hstep(t0, asl, 0);
      hstep(t0, asl, 1);
      hstep(t1, asl + 32, 0);
      hstep(t1, asl + 32, 1);
      __syncwarp();   // every lane is done with both stages and both slices
      if (lane == 0) {
        mbar_arrive(empty0 + 8 * s0);
        mbar_arrive(empty0 + 8 * s1);
      }
      return true;
    };

    // two register sets, so that no load result is moved before it is used
    load_scale(0, qa, sa);
    load_scale(1, qb, sb);
    named_barrier_sync(1, kGvConsumers * 32);   // level table complete
    int i = 0;
    for (; i + 1 < nstage; i += 2)
      if (!stage2(i)) break;
    // an odd last weight stage, then the adapter stages, one at a time
    for (bool ok = i + 1 >= nstage; ok && i < nall; ++i) ok = stage(i, (i & 1) ? qb : qa, (i & 1) ? sb : sa);
  }
  __syncthreads();   // ring no longer read or written: it becomes the partial buffer

  // D fragment of tile j: column 8g+2j (c[0], c[1]) and 8g+2j+1 (c[2], c[3]) of the
  // group, tokens 2t and 2t+1 of token tile a.  Row half 1 stores, row half 0 adds:
  // the CTA's partial of the tile, [M][256] fp32.
  for (int pass = 1; pass >= 0; --pass) {
    if (warp < kGvConsumers && half == pass) {
#pragma unroll
      for (int a = 0; a < MT; ++a)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int m = a * 8 + 2 * t + q;
            if (m < p.M) {
              float2* dst = reinterpret_cast<float2*>(part + m * kTileCols + cg * 64 + 8 * g + 2 * j);
              float2 v = make_float2(acc[a][j][q], acc[a][j][2 + q]);
              if (pass == 0) {
                const float2 o = *dst;
                v.x += o.x;
                v.y += o.y;
              }
              *dst = v;
            }
          }
    }
    __syncthreads();
  }

  // ---------------------------------------------------------------- cluster reduction
  // CTA o of the cluster owns the tile's 4-column groups [o * cap, (o + 1) * cap);
  // every CTA stores its partial of each group into the owner's receive buffer
  // (slot = its rank), and after one cluster barrier each owner adds its S
  // slots in split order (the result does not depend on timing).
  const int S = static_cast<int>(cluster_nctarank()), rank = static_cast<int>(cluster_ctarank());
  const int groups = p.M * (kTileCols / 4);
  const int cap = (groups + S - 1) / S;
  const uint32_t recv_addr = smem_addr(recv);
  for (int q = tid; q < groups; q += kGvThreads) {
    const int o = q / cap, slot = q - o * cap;
    const float4 v = *reinterpret_cast<const float4*>(part + 4 * q);
    st_shared_cluster_v4(mapa_shared(recv_addr + static_cast<uint32_t>((rank * cap + slot) * 16), o), v);
  }
  cluster_sync();   // every push of every split has landed
  for (int slot = tid; slot < cap && rank * cap + slot < groups; slot += kGvThreads) {
    const int q = rank * cap + slot;
    float4 y = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int sp = 0; sp < S; ++sp) {
      const float4 v = reinterpret_cast<const float4*>(recv)[sp * cap + slot];
      y.x += v.x;
      y.y += v.y;
      y.z += v.z;
      y.w += v.w;
    }
    const int m = q / (kTileCols / 4), c4 = (q % (kTileCols / 4)) * 4;
    const int64_t col = col0 + c4;
    if (col < p.N)
      *reinterpret_cast<uint2*>(p.Y + static_cast<int64_t>(m) * p.N + col) =
          make_uint2(pack_bf16x2(y.x, y.y), pack_bf16x2(y.z, y.w));
  }
}

// + 1 KB to align the ring to the swizzle atom
constexpr size_t kGvSmemBytes = 1024 + kGvStages * kStageBytes + kLutBytes + kGvConsumers * 64 * 4 + kRecvBytes;

// Clusters of each size (1 .. kMaxCluster CTAs) that can be resident at once,
// queried once per device (the kernels' attributes are set on the way); all
// zero if the device cannot run the kernel.  `sms`: the device's SM count.
struct ClusterFit {
  int max_active[kMaxCluster + 1];
  int sms;
};

const ClusterFit& cluster_fit() {
  static std::mutex mu;
  static ClusterFit fits[64];
  static bool done[64] = {};
  static const ClusterFit none{};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return none;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return fits[dev];
  ClusterFit f{};
  bool ok = true;
  for (auto fn : {nf4_gemv_kernel<1>, nf4_gemv_kernel<2>}) {
    ok = ok && cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(kGvSmemBytes)) == cudaSuccess;
    ok = ok && cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  }
  for (int S = 1; ok && S <= kMaxCluster; ++S) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(1, S);
    cfg.blockDim = dim3(kGvThreads);
    cfg.dynamicSmemBytes = kGvSmemBytes;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = S;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n1 = 0, n2 = 0;
    if (cudaOccupancyMaxActiveClusters(&n1, nf4_gemv_kernel<1>, &cfg) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n2, nf4_gemv_kernel<2>, &cfg) != cudaSuccess)
      break;
    f.max_active[S] = n1 < n2 ? n1 : n2;
  }
  if (cudaDeviceGetAttribute(&f.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) f.sms = 0;
  cudaGetLastError();
  fits[dev] = f;
  done[dev] = true;
  return fits[dev];
}

// K-splits S (the cluster size) and rows per split Kc for a K x N weight at M
// tokens, fewer splits on a tie.  False if no cluster size fits.
//   * M <= 8: the split that minimises waves x rows per CTA.  A CTA streams its
//     stages at about the same rate whether or not it shares its SM, so more
//     CTAs stream more at once.
//   * M > 8 (two token tiles, twice the products per stage): the consumer warps
//     are issue-bound and an SM streams at about the same rate with one CTA or
//     two; a CTA alone on its SM takes a stage in about 7/13 of the time two CTAs
//     sharing an SM take.  The split minimises the stages an SM streams: a wave
//     of more CTAs than SMs puts two on some SMs, and those set its length.
// (Both rules measured on the 4096 x 4096 weight: at M = 1, 8 splits of 8 stages
// take 11.7 us per forward against 9.6 us for 13 splits of 5; at M = 16, 15.6
// against 17.0 us.)
bool gemv_plan(int64_t K, int64_t N, int64_t M, const ClusterFit& fit, int& S, int& Kc) {
  const int64_t tiles = (N + kTileCols - 1) / kTileCols;
  const int64_t stages = K / kStageRows;
  int64_t best_cost = -1;
  for (int s = 1; s <= kMaxCluster && s <= stages; ++s) {
    if (fit.max_active[s] < 1) continue;
    const int64_t kc = ((K + s - 1) / s + kStageRows - 1) / kStageRows * kStageRows;
    if ((K + kc - 1) / kc != s) continue;   // another s gives the same split
    const int64_t waves = (tiles + fit.max_active[s] - 1) / fit.max_active[s];
    const int64_t wave_ctas = (tiles < fit.max_active[s] ? tiles : fit.max_active[s]) * s;
    const int64_t cost = M <= 8 ? waves * kc : waves * (kc / kStageRows) * (wave_ctas > fit.sms ? 13 : 7);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      S = s;
      Kc = static_cast<int>(kc);
    }
  }
  return best_cost >= 0;
}

PFN_cuTensorMapEncodeTiled_v12000 gemv_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

}  // namespace

bool gemv_supported(int64_t M, int64_t K, int64_t N) {
  int S, Kc;
  return M >= 1 && M <= kGemvMaxTokens && gemv_plan(K, N, M, cluster_fit(), S, Kc);
}

cudaError_t launch_gemv(const WeightView& w, const uint16_t* X, const uint16_t* V, const uint16_t* B, int64_t M,
                        int r, uint16_t* Y, uint32_t* status, cudaStream_t stream) {
  int S, Kc;
  if (w.fmt == kFmtInt16 || M < 1 || M > kGemvMaxTokens || !gemv_plan(w.in, w.out, M, cluster_fit(), S, Kc))
    return cudaErrorInvalidValue;   // NF4 weights only
  auto enc = gemv_encoder();
  if (!enc) return cudaErrorInvalidValue;
  // codes as an (in x out/2) byte matrix; box = one 256-column tile (128 bytes) x 64 rows
  CUtensorMap tm;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(w.out / 2), static_cast<cuuint64_t>(w.in)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(w.out / 2)};
  cuuint32_t box[2] = {128, kStageRows};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(w.codes), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // X (M x in) bf16: box = 64 columns (128 bytes) x M rows
  CUtensorMap tx;
  cuuint64_t xdims[2] = {static_cast<cuuint64_t>(w.in), static_cast<cuuint64_t>(M)};
  cuuint64_t xstrides[1] = {static_cast<cuuint64_t>(w.in * 2)};
  cuuint32_t xbox[2] = {kStageRows, static_cast<cuuint32_t>(M)};
  if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), xdims, xstrides, xbox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // B (r x out) bf16: box = 64 columns (128 bytes) x 16 adapter rows
  CUtensorMap tb;
  cuuint64_t bdims[2] = {static_cast<cuuint64_t>(w.out), static_cast<cuuint64_t>(r)};
  cuuint64_t bstrides[1] = {static_cast<cuuint64_t>(w.out * 2)};
  cuuint32_t bbox[2] = {64, 16};
  if (enc(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(B), bdims, bstrides, bbox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // V (M x r) bf16: box = 16 adapter columns (32 bytes) x M rows
  CUtensorMap tv;
  cuuint64_t vdims[2] = {static_cast<cuuint64_t>(r), static_cast<cuuint64_t>(M)};
  cuuint64_t vstrides[1] = {static_cast<cuuint64_t>(r * 2)};
  cuuint32_t vbox[2] = {16, static_cast<cuuint32_t>(M)};
  if (enc(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(V), vdims, vstrides, vbox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  GemvArgs a{w.dq_codes, w.dq_scales, w.in, w.out, static_cast<int>(M), r, Y, Kc, status, w.fmt == kFmtU8 ? 1 : 0};

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>((w.out + kTileCols - 1) / kTileCols), static_cast<unsigned>(S));
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = kGvSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = static_cast<unsigned>(S);
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  timing_before(QLORA_KERNEL_GEMV, stream);
  const cudaError_t e = M <= 8 ? cudaLaunchKernelEx(&cfg, nf4_gemv_kernel<1>, tm, tx, tb, tv, a)
                               : cudaLaunchKernelEx(&cfg, nf4_gemv_kernel<2>, tm, tx, tb, tv, a);
  timing_after(QLORA_KERNEL_GEMV, stream);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace qlora
