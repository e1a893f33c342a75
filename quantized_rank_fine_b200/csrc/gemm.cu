// Fused dequant GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM), for
// NF4 weights (one absmax per 64 weights, E4M3 or linear uint8 codes) and for the
// symmetric INT weights of qlora_quantize_int (one fp32 scale per 16 weights).
//
//   forward  Y  = [X | V] . [deq(Wq) ; B]      (M x out, K = in + r)
//   dX       dX = [dY | U] . [deq(Wq)^T ; A^T] (M x in,  K = out + r)
//
// ("How it works" steps 2-4 and "What QLoRA adds over LoRA" of "QLoRA (low-rank
// adapters on a quantized model)": the frozen weight is dequantised to bf16 for
// each matmul; the adapter product (X A) B, and U A^T in the backward, is the
// same contraction extended by r along K, so it lands in the same accumulator.)
//
// Pair tile 512 (M) x 256 (N), K step 64, computed by two CTAs on the two SMs of
// a cluster of 2 with the pair form of the tensor-core MMA (tcgen05 cta_group::2):
// one M=256 x N=256 MMA reads 128 rows of A and 128 columns of B from each CTA's
// shared memory and writes each CTA's 128 rows into its own TMEM.  Two such
// MMAs per K-step (pair rows 0-255 and 256-511) fill each CTA's 512 TMEM
// columns, so a CTA holds 256 output rows x 256 columns, yet dequantises only
// its own 128 columns of the weight tile: each weight is dequantised M/512
// times, and a CTA's shared-memory stage is 52 KB (A 32 KB, its dequantised B
// half 16 KB, codes 4 KB), which leaves room for a 4-deep ring.
// Warp roles (320 threads per CTA):
//   warp 0     TMA producer (both CTAs): per K-step the CTA's two 128-row
//              activation boxes (128B swizzle) and the packed codes of its
//              half of the weight tile; for the adapter K-steps the V/U rows and
//              the CTA's half of the B / A^T tile instead.
//   warp 1     TMEM allocation (both CTAs, pair form); in the even CTA of the
//              pair the single thread that issues the MMAs for both.
//   warps 2-9  dequant producers, two groups of 4 warps taking alternate
//              K-steps (one thread per 64 weights per step): codes from shared
//              memory -> 16-entry bf16 table per 64-weight block (NF4) or per
//              16-weight group (INT) -> byte-permute lookup -> 16-byte stores in
//              the UMMA canonical layout; then the epilogue, all 8 warps:
//              TMEM -> registers -> bf16 -> a 32 x 32 block in shared memory
//              (64-byte swizzle) -> one TMA tensor store per block, so every
//              output line is written whole.  The staging blocks live in the
//              dequantised-weight regions of the ring, which no one else
//              touches while the dequant warps run the epilogue.
// Barriers per stage: `loaded` (this CTA's TMA bytes), `ready` (in the even CTA:
// the 4 dequant warps of each CTA that took the stage, each after its CTA's
// stage has landed and its weight half is written) and `free` (the pair MMAs'
// commit, multicast to both CTAs); per work item `tmem_full` (the last MMA's
// commit, multicast) and `tmem_empty` (in the even CTA: the 8 epilogue warps of
// each CTA have read their TMEM).
// The weight tile is written MN-major for the forward (N contiguous in W) and
// K-major for dX (K contiguous in W), so the dequant never transposes.
//
// Schedule (persistent grid, one pair per two SMs).  A tile's K-steps are the
// weight steps followed by the adapter steps, S in all.  The first `dp_tiles`
// tiles are whole work items dealt round robin over the pairs; the K-steps of
// the remaining `sk_tiles` tiles are laid end to end and cut into one
// contiguous range per pair ("stream-K"), so that every pair does the same
// number of K-steps when the tile count is not a multiple of the pair count.
// A range that starts inside a tile leaves a partial accumulator: each CTA of
// that pair stores its half (fp32) in its own slot of the workspace and counts
// its warps into the slot's counter.  The pair whose range holds the tile's
// first K-step owns the tile: it reaches that item last in its own range, waits
// for the counters of the pairs after it that hold the rest of the tile, adds
// their slots in pair order (deterministic) and writes the output.  A pair's
// first item is the only one that can leave a partial and its last the only one
// that can wait, so the waits form no cycle; they are bounded like every other
// wait.  The owner clears the counters it consumed before it exits, so they are
// zero for the next launch.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

#include <cudaTypedefs.h>

namespace qlora {

namespace {

using namespace sm100;

constexpr int kPairM = 512;                      // rows of a pair tile
constexpr int kBM = 256;                         // rows per CTA (two 128-row accumulators)
constexpr int kBN = 256;                         // columns of a pair tile
constexpr int kHalfN = 128;                      // columns each CTA dequantises
constexpr int kBK = 64, kStages = 4;
constexpr int kThreads = 320;
constexpr int kDeqWarps = 8;
constexpr uint32_t kABytes = kBM * kBK * 2;      // 32 KB: two 128-row boxes
constexpr uint32_t kBBytes = kHalfN * kBK * 2;   // 16 KB: this CTA's dequantised half
constexpr uint32_t kCBytes = kHalfN * kBK / 2;   // 4 KB of packed codes
constexpr uint32_t kStageBytes = kABytes + kBBytes + kCBytes;
constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024 + 256;
constexpr uint32_t kTmemCols = 512;

struct GemmArgs {
  const uint8_t* codes;
  const uint8_t* dq_codes;
  const float* dq_scales;
  int64_t w_out;      // columns of the stored weight (out)
  int64_t M, N, K;    // output M x N, weight reduction length K (multiple of 64)
  int r;
  uint16_t* D;        // bf16 (M, N)
  uint32_t* status;
  int dq_u8;          // absmax codes are linear uint8 (else E4M3)
  // schedule (see the file header)
  int tiles_n;        // pair tiles along N; tile t covers rows (t / tiles_n) * 512, columns (t % tiles_n) * 256
  int dp_tiles;       // tiles [0, dp_tiles): whole items, round robin over the pairs
  int sk_tiles;       // tiles [dp_tiles, dp_tiles + sk_tiles): K-steps split evenly over the pairs
  float* partials;    // gridDim.x slots (one per CTA) of 256 x 256 fp32 (used when sk_tiles > 0)
  uint32_t* counters; // gridDim.x counters, zero at launch (used when sk_tiles > 0)
};

constexpr uint32_t kSlotFloats = kBM * kBN;    // one CTA's partial accumulator (256 KB)

// One work item: K-steps [kb0, kb1) of tile `tile`; `sk` is its index within the
// split region, or -1 for a whole tile.
struct WorkItem {
  int tile, kb0, kb1, sk;
};

// First K-step (in the split region's flattened numbering) of pair c's range.
__device__ __forceinline__ int64_t sk_range_start(int64_t units, int c) {
  return units * c / static_cast<int64_t>(gridDim.x >> 1);
}

// Item i of this CTA's pair; false once the pair has no more.
__device__ __forceinline__ bool work_item(const GemmArgs& p, int S, int i, WorkItem& w) {
  const int G = gridDim.x >> 1, b = blockIdx.x >> 1;
  const int n_dp = p.dp_tiles > b ? (p.dp_tiles - b + G - 1) / G : 0;
  if (i < n_dp) {
    w.tile = b + i * G;
    w.kb0 = 0;
    w.kb1 = S;
    w.sk = -1;
    return true;
  }
  if (p.sk_tiles == 0) return false;
  const int64_t units = static_cast<int64_t>(p.sk_tiles) * S;
  const int64_t s0 = sk_range_start(units, b), s1 = sk_range_start(units, b + 1);
  const int64_t t = s0 / S + (i - n_dp);
  if (s0 >= s1 || t * S >= s1) return false;
  w.sk = static_cast<int>(t);
  w.tile = p.dp_tiles + w.sk;
  w.kb0 = static_cast<int>(s0 > t * S ? s0 - t * S : 0);
  w.kb1 = static_cast<int>(s1 - t * S < S ? s1 - t * S : S);
  return true;
}

// Pairs b+1 .. (return value - 1) hold the rest of split tile `sk` owned by pair b.
__device__ __forceinline__ int sk_contributors_end(int64_t units, int S, int sk, int b) {
  int c = b + 1;
  const int64_t tile_end = static_cast<int64_t>(sk + 1) * S;
  while (c < static_cast<int>(gridDim.x >> 1) && sk_range_start(units, c) < tile_end) ++c;
  return c;
}

// Per-block table: v_j = bf16(fl32(level_j * a)) for j = 0..15, split into the
// low bytes (lo[0..3]) and high bytes (hi[0..3]) of the 16 entries, 4 per word.
struct BlockLut {
  uint32_t lo[4], hi[4];
};

// Level j of the weight format: the NF4 level, or the integer j - 8 of the
// symmetric INT format (qlora_quantize_int).
template <bool kInt>
__device__ __forceinline__ constexpr float format_level(int j) {
  return kInt ? static_cast<float>(j - 8) : nf4_level(j);
}

template <bool kInt>
__device__ __forceinline__ BlockLut make_lut(float a) {
  uint32_t pr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    pr[i] = pack_bf16x2(mul_rn(format_level<kInt>(2 * i), a), mul_rn(format_level<kInt>(2 * i + 1), a));
  BlockLut t;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    t.lo[q] = __byte_perm(pr[2 * q], pr[2 * q + 1], 0x6420);
    t.hi[q] = __byte_perm(pr[2 * q], pr[2 * q + 1], 0x7531);
  }
  return t;
}

// Four 4-bit codes (nibbles of x, element order low to high) -> two bf16x2 words.
__device__ __forceinline__ void lut4(const BlockLut& t, uint32_t x, uint32_t& o01, uint32_t& o23) {
  const uint32_t s_lo = x & 0x7777u;                              // index within a half table
  const uint32_t s_pick = 0x3210u | ((x >> 1) & 0x4444u);         // +4 where the code is >= 8
  const uint32_t lo = __byte_perm(__byte_perm(t.lo[0], t.lo[1], s_lo),
                                  __byte_perm(t.lo[2], t.lo[3], s_lo), s_pick);
  const uint32_t hi = __byte_perm(__byte_perm(t.hi[0], t.hi[1], s_lo),
                                  __byte_perm(t.hi[2], t.hi[3], s_lo), s_pick);
  o01 = __byte_perm(lo, hi, 0x5140);
  o23 = __byte_perm(lo, hi, 0x7362);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// Scale data of one K-step for a dequant thread: the absmax code and group
// scale of its 64-weight NF4 block, or the four fp32 scales of its four
// 16-weight groups (INT16 format).
template <bool kInt>
struct ScaleSlot {
  uint8_t c = 0;
  float s = 0.0f;
};
template <>
struct ScaleSlot<true> {
  float4 s = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
};

template <bool kDX, bool kInt>
__global__ void __launch_bounds__(kThreads, 1)
nf4_gemm_kernel(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_ext_a,
                const __grid_constant__ CUtensorMap tm_ext_b, const __grid_constant__ CUtensorMap tm_codes,
                const __grid_constant__ CUtensorMap tm_out, const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * kStages + 4);
  const uint32_t loaded0 = smem_addr(bars), ready0 = smem_addr(bars + kStages);
  const uint32_t free0 = smem_addr(bars + 2 * kStages), tmem_full = smem_addr(bars + 3 * kStages);
  const uint32_t tmem_empty = smem_addr(bars + 3 * kStages + 1);
  const uint32_t mma_drained = smem_addr(bars + 3 * kStages + 2);
  // the 8 epilogue warps of this CTA are done staging an item's output in the
  // dequantised-weight regions (they may then be refilled)
  const uint32_t staging_free = smem_addr(bars + 3 * kStages + 3);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();         // 0: issues the pair's MMAs
  const int nkb_w = static_cast<int>(p.K / kBK);
  const int n_ext = (p.r + kBK - 1) / kBK;
  const int S = nkb_w + n_ext;                     // K-steps per tile
  const int64_t sk_units = static_cast<int64_t>(p.sk_tiles) * S;

  if (threadIdx.x == 0) {
    // `ready` and `tmem_empty` are used in the even CTA: a stage's `ready`
    // counts the 4 dequant warps of each CTA that took it, `tmem_empty` all 8
    // epilogue warps of each CTA
    for (int s = 0; s < kStages; ++s) {
      mbar_init(loaded0 + 8 * s, 1);
      mbar_init(ready0 + 8 * s, kDeqWarps);          // 4 warps of each CTA per stage
      mbar_init(free0 + 8 * s, 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 2 * kDeqWarps);
    mbar_init(mma_drained, 1);
    mbar_init(staging_free, kDeqWarps);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_act);
    tma_prefetch_desc(&tm_ext_a);
    tma_prefetch_desc(&tm_ext_b);
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_out);
  }
  // both CTAs' barriers initialised and TMEM allocated before any cross-CTA use
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the even CTA's barriers, as seen from either CTA of the pair
  const uint32_t ready_lead = mapa_shared(ready0, 0);
  const uint32_t tmem_empty_lead = mapa_shared(tmem_empty, 0);
  // Launched as a programmatic dependent of the rank-r kernel of the same call
  // (V before the forward, U or dA/dB before dX).  That kernel lets this one start
  // only after its own wait for the kernel before it, so everything this kernel
  // reads except that kernel's output (V or U, read by the adapter steps) is
  // final: the activations and weights stream at once, and only the adapter
  // steps and the first global write wait for the rank-r kernel to finish.
  grid_launch_dependents();

  int owned_end = 0;    // > 0: this pair owns a split tile whose other parts pairs b+1 .. owned_end-1 hold

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int g = 0;        // K-steps issued so far (ring position)
      int sf_done = 0;  // epilogues (staging_free phases) seen complete
      bool alive = true;
      WorkItem w;
      for (int it = 0; alive && work_item(p, S, it, w); ++it) {
        const int32_t ma = (w.tile / p.tiles_n) * kPairM + kHalfN * static_cast<int32_t>(rank);
        const int32_t nh = (w.tile % p.tiles_n) * kBN + kHalfN * static_cast<int32_t>(rank);
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++g) {
          const int s = g % kStages;
          const uint32_t ph = (g / kStages) & 1;
          if (!mbar_wait(free0 + 8 * s, ph ^ 1, p.status, kFlagTimeoutProducer)) {
            alive = false;
            break;
          }
          const uint32_t a_dst = smem_addr(smem + s * kStageBytes);
          const uint32_t b_dst = a_dst + kABytes;
          const uint32_t c_dst = b_dst + kBBytes;
          const uint32_t bar = loaded0 + 8 * s;
          if (kb < nkb_w) {
            mbar_arrive_expect_tx(bar, kABytes + kCBytes);
            tma_load_2d(a_dst, &tm_act, bar, kb * kBK, ma);
            tma_load_2d(a_dst + kABytes / 2, &tm_act, bar, kb * kBK, ma + kBM);
            if (!kDX) tma_load_2d(c_dst, &tm_codes, bar, nh / 2, kb * kBK);
            else tma_load_2d(c_dst, &tm_codes, bar, kb * (kBK / 2), nh);
          } else {
            const int j = kb - nkb_w;
            grid_dependency_wait();   // V or U is written by the kernel before
            // the adapter's weight tile lands in the dequantised-weight region,
            // which the previous item's epilogue may still use as output staging:
            // wait for the epilogues of items 0 .. it-1, phase by phase (in order,
            // so that no parity is mistaken for the one two phases later)
            bool ok = true;
            for (; ok && sf_done < it; ++sf_done)
              ok = mbar_wait(staging_free, static_cast<uint32_t>(sf_done & 1), p.status, kFlagTimeoutProducer);
            if (!ok) {
              alive = false;
              break;
            }
            mbar_arrive_expect_tx(bar, kABytes + kBBytes);
            tma_load_2d(a_dst, &tm_ext_a, bar, j * kBK, ma);
            tma_load_2d(a_dst + kABytes / 2, &tm_ext_a, bar, j * kBK, ma + kBM);
            if (!kDX) {
              tma_load_2d(b_dst, &tm_ext_b, bar, nh, j * kBK);
              tma_load_2d(b_dst + 8192, &tm_ext_b, bar, nh + 64, j * kBK);
            } else {
              tma_load_2d(b_dst, &tm_ext_b, bar, j * kBK, nh);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(256, 256, false, !kDX);
      int g = 0;
      bool alive = true;
      WorkItem w;
      for (int it = 0; alive && work_item(p, S, it, w); ++it) {
        // both CTAs' epilogues must have read the previous item's accumulators
        if (it > 0 && !mbar_wait(tmem_empty, (it - 1) & 1, p.status, kFlagTimeoutMma)) break;
        tc_fence_after();
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++g) {
          const int s = g % kStages;
          const uint32_t ph = (g / kStages) & 1;
          // `ready` completes once both CTAs' dequant warps have seen their
          // stage land and written their weight halves
          if (!mbar_wait(ready0 + 8 * s, ph, p.status, kFlagTimeoutMma) ||
              !mbar_wait(loaded0 + 8 * s, ph, p.status, kFlagTimeoutMma)) {
            alive = false;
            break;
          }
          tc_fence_after();
          int nk16 = 4;
          if (kb >= nkb_w) nk16 = min(4, (p.r - (kb - nkb_w) * kBK + 15) / 16);
          const uint32_t a_base = smem_addr(smem + s * kStageBytes);
          const uint32_t b_base = a_base + kABytes;
          for (int kk = 0; kk < nk16; ++kk) {
            const uint64_t bdesc = kDX ? smem_desc_sw128(b_base + kk * 32, 16, 1024)
                                       : smem_desc_sw128(b_base + kk * 2048, 8192, 1024);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t adesc = smem_desc_sw128(a_base + h * (kABytes / 2) + kk * 32, 16, 1024);
              umma_bf16_pair(tmem_base + h * 256, adesc, bdesc, idesc, (kb != w.kb0 || kk != 0) ? 1u : 0u);
            }
          }
          umma_commit_pair_multicast(free0 + 8 * s, 0x3);
        }
        if (alive) umma_commit_pair_multicast(tmem_full, 0x3);
      }
      // every MMA issued (also on a path that gave up) has completed before
      // the pair's TMEM can be freed
      umma_commit_pair_multicast(mma_drained, 0x1);
      mbar_wait(mma_drained, 0, p.status, kFlagTimeoutMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequant producers + epilogue
    // The 8 warps form two groups of 4 that take alternate K-steps (group 0 the
    // even stage counts, group 1 the odd ones), so each group has two pipeline
    // periods per stage; within a group each thread dequantises one whole
    // 64-weight block of the CTA's half tile (one table per block).
    const int group = (warp - 2) >> 2;
    const int t = threadIdx.x - 64 - 128 * group;   // 0..127
    const int64_t blocks_per_row = p.w_out / kBlock;
    int kr = 0, j = 0, nr = 0;
    uint32_t row_off, code_off0, code_off1;
    int swz;
    if (!kDX) {
      // Quarter-warps (8 lanes) take 8 consecutive k rows of one 64-wide n
      // block, so their 16-byte stores fall in 8 distinct bank groups.
      kr = (t & 7) + (((t >> 3) & 7) << 3);        // 0..63
      j = t >> 6;                                   // which 64-wide n block of the half
      row_off = j * 8192 + (kr >> 3) * 1024 + (kr & 7) * 128;
      swz = kr & 7;
      // codes tile: 64 rows of 64 bytes, 64-byte swizzle (16-byte chunk ^ (row >> 1) & 3)
      code_off0 = kr * 64 + (((2 * j) ^ ((kr >> 1) & 3)) << 4);
      code_off1 = kr * 64 + (((2 * j + 1) ^ ((kr >> 1) & 3)) << 4);
    } else {
      nr = t;                                       // n row of the half tile, 0..127
      row_off = nr * 128;
      swz = nr & 7;
      // codes tile: 128 rows of 32 bytes, 32-byte swizzle (16-byte chunk ^ (row >> 2) & 1)
      code_off0 = nr * 32 + ((0 ^ ((nr >> 2) & 1)) << 4);
      code_off1 = nr * 32 + ((1 ^ ((nr >> 2) & 1)) << 4);
    }
    // K-step kb moves the block index by 64 rows (forward) or 1 block (dX).
    const int64_t blk_step = kDX ? 1 : 64 * blocks_per_row;
    // epilogue: this thread's accumulator row and TMEM address
    const int quarter = warp & 3;                   // TMEM lanes 32*quarter .. +31
    const int half = (warp - 2) >> 2;               // which accumulator (pair rows 0-255 or 256-511)
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + half * 256;
    // float4 index of this thread's first chunk within a partial slot: chunk q
    // of column block cb sits at ((cb * 2 + half) * 4 + quarter) * 256 + q * 32 + lane,
    // so each warp store covers 512 contiguous bytes
    const uint32_t slot_lane = ((half * 4 + quarter) * 8) * 32 + lane;
    // this warp's two 2 KB output staging blocks: in the dequantised-weight
    // region of stage (warp - 2) / 2, the warp's half of it
    const uint32_t stage_out = smem_addr(smem + ((warp - 2) >> 1) * kStageBytes + kABytes) +
                               static_cast<uint32_t>((warp - 2) & 1) * (kBBytes / 2);

    int g = 0;
    bool alive = true;
    WorkItem w;
    for (int it = 0; alive && work_item(p, S, it, w); ++it) {
      const int64_t m0 = static_cast<int64_t>(w.tile / p.tiles_n) * kPairM;
      const int64_t n0 = static_cast<int64_t>(w.tile % p.tiles_n) * kBN;
      const int64_t nh = n0 + kHalfN * rank;
      bool valid;
      int64_t blk;                                  // block index at kb = 0
      if (!kDX) {
        valid = (nh + 64 * j) < p.N;
        blk = static_cast<int64_t>(kr) * blocks_per_row + (nh >> 6) + j;
      } else {
        valid = (nh + nr) < p.N;
        blk = (nh + nr) * blocks_per_row;
      }
      // This group's K-steps of the item: those whose stage count has its parity.
      const int g0 = g;
      const int kb_first = w.kb0 + ((group - g0) & 1);
      g += w.kb1 - w.kb0;
      // Scale data of the group's next K-steps, loaded two of its steps ahead
      // into one of two register slots; the loop is unrolled by two so that a
      // slot is consumed and refilled in place (moving a pending load's
      // register to another would wait for the load one step early).
      auto load_slot = [&](int kb, ScaleSlot<kInt>& sl) {
        if (!valid || kb >= nkb_w) return;
        const int64_t b = blk + kb * blk_step;
        if constexpr (kInt) {
          sl.s = __ldg(reinterpret_cast<const float4*>(p.dq_scales) + b);
        } else {
          sl.c = __ldg(p.dq_codes + b);
          sl.s = __ldg(p.dq_scales + b / kGroup);
        }
      };
      ScaleSlot<kInt> slotA, slotB;
      load_slot(kb_first, slotA);
      load_slot(kb_first + 2, slotB);
      // one K-step with its scale data in `sl`; refills it for kb + 4
      auto step = [&](int kb, ScaleSlot<kInt>& sl) -> bool {
        const int gg = g0 + (kb - w.kb0);
        const int s = gg % kStages;
        const uint32_t ph = (gg / kStages) & 1;
        // every lane waits; the warp leaves the loop together if the wait gave up
        const bool got = mbar_wait(loaded0 + 8 * s, ph, p.status, kFlagTimeoutProducer);
        if (!__all_sync(0xffffffffu, got)) return false;
        if (kb < nkb_w) {
          const uint32_t stage = smem_addr(smem + s * kStageBytes);
          const uint32_t dst = stage + kABytes + row_off;
          const uint32_t csrc = stage + kABytes + kBBytes;
          uint32_t wd[8];
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(wd[0]), "=r"(wd[1]), "=r"(wd[2]), "=r"(wd[3]) : "r"(csrc + code_off0));
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(wd[4]), "=r"(wd[5]), "=r"(wd[6]), "=r"(wd[7]) : "r"(csrc + code_off1));
          // one table per block (NF4) or per 16-weight group (INT16, words 2q, 2q+1)
          BlockLut lut[kInt ? 4 : 1];
          if constexpr (kInt) {
            lut[0] = make_lut<true>(valid ? sl.s.x : 0.0f);
            lut[1] = make_lut<true>(valid ? sl.s.y : 0.0f);
            lut[2] = make_lut<true>(valid ? sl.s.z : 0.0f);
            lut[3] = make_lut<true>(valid ? sl.s.w : 0.0f);
          } else {
            lut[0] = make_lut<false>(valid ? absmax_deq(sl.c, sl.s, p.dq_u8 != 0) : 0.0f);
          }
          load_slot(kb + 4, sl);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const BlockLut& L = lut[kInt ? c >> 1 : 0];
            uint32_t o0, o1, o2, o3;
            lut4(L, wd[c] & 0xFFFFu, o0, o1);
            lut4(L, wd[c] >> 16, o2, o3);
            st_shared_v4(dst + ((c ^ swz) << 4), o0, o1, o2, o3);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(ready_lead + 8 * s);
        return true;
      };
      for (int kb = kb_first; kb < w.kb1; kb += 4) {
        if (!step(kb, slotA) || (kb + 2 < w.kb1 && !step(kb + 2, slotB))) {
          alive = false;
          break;
        }
      }
      if (!alive) break;

      // ---------------------------------------------------------- epilogue of the item
      grid_dependency_wait();   // no global write before the kernel before has finished
      if (!__all_sync(0xffffffffu, mbar_wait(tmem_full, it & 1, p.status, kFlagTimeoutEpilogue))) break;
      tc_fence_after();
      if (w.kb0 > 0) {
        // the rest of a split tile: fp32 partial into this CTA's slot
        float4* slot = reinterpret_cast<float4*>(p.partials) + static_cast<size_t>(blockIdx.x) * (kSlotFloats / 4);
#pragma unroll 1
        for (int cb = 0; cb < kBN / 32; ++cb) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + cb * 32, v);   // returns once the values are in v
          float4* dst = slot + cb * 2048 + slot_lane;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            __stcg(dst + q * 32, make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                             __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3])));
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_gpu_add(p.counters + blockIdx.x, 1);
      } else {
        // a whole tile, or the head of a split tile plus the other pairs' partials
        const int pair = blockIdx.x >> 1;
        int c_end = pair + 1;
        bool have = true;
        if (w.kb1 < S) {
          c_end = sk_contributors_end(sk_units, S, w.sk, pair);
          owned_end = c_end;
          for (int c = pair + 1; c < c_end; ++c)
            have = have && wait_counter(p.counters + 2 * c + rank, kDeqWarps, p.status, kFlagTimeoutEpilogue);
        }
        // the warp's 32 rows; each 32-column block goes out through shared
        // memory as one TMA store (rows and columns past the output are clipped)
        const int64_t row0 = m0 + half * kBM + kHalfN * rank + quarter * 32;
        // The other pairs' partials of column block cb, summed in pair order; the
        // first pair's values are only loaded here and added one block later, so
        // their L2 round trip overlaps the previous block's store.
        const bool merge = have && c_end > pair + 1;
        float4 pre[8];
        auto fetch = [&](int cb) {
          const float4* src = reinterpret_cast<const float4*>(p.partials) +
                              static_cast<size_t>(2 * (pair + 1) + rank) * (kSlotFloats / 4) + cb * 2048 + slot_lane;
#pragma unroll
          for (int q = 0; q < 8; ++q) pre[q] = __ldcg(src + q * 32);
        };
        if (merge) fetch(0);
#pragma unroll 1
        for (int cb = 0; cb < kBN / 32; ++cb) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + cb * 32, v);   // returns once the values are in v
          float acc[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = __uint_as_float(v[i]);
          if (merge) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              acc[4 * q] += pre[q].x;
              acc[4 * q + 1] += pre[q].y;
              acc[4 * q + 2] += pre[q].z;
              acc[4 * q + 3] += pre[q].w;
            }
            for (int c = pair + 2; c < c_end; ++c) {
              const float4* src = reinterpret_cast<const float4*>(p.partials) +
                                  static_cast<size_t>(2 * c + rank) * (kSlotFloats / 4) + cb * 2048 + slot_lane;
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 x = __ldcg(src + q * 32);
                acc[4 * q] += x.x;
                acc[4 * q + 1] += x.y;
                acc[4 * q + 2] += x.z;
                acc[4 * q + 3] += x.w;
              }
            }
            if (cb + 1 < kBN / 32) fetch(cb + 1);
          }
          const int64_t col = n0 + cb * 32;
          // Only blocks that are stored touch the staging buffers, so that every
          // write to a buffer follows the commit of the store that last read it
          // (the blocks past the output's last column or row are a suffix of the
          // warp's blocks and are skipped whole).
          if (row0 >= p.M || col >= p.N) continue;
          const uint32_t buf = stage_out + static_cast<uint32_t>(cb & 1) * 2048u;
          // the store issued from this buffer two blocks ago has read it
          if (lane == 0 && cb >= 2) bulk_wait_read<1>();
          __syncwarp();
          // row `lane` of the block, 64 bytes as four 16-byte chunks, chunk c at
          // c ^ ((row >> 1) & 3) (the 64-byte swizzle of the tensor map)
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_v4(buf + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4), pack_bf16x2(acc[8 * q + 0], acc[8 * q + 1]),
                         pack_bf16x2(acc[8 * q + 2], acc[8 * q + 3]), pack_bf16x2(acc[8 * q + 4], acc[8 * q + 5]),
                         pack_bf16x2(acc[8 * q + 6], acc[8 * q + 7]));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tm_out, buf, static_cast<int32_t>(col), static_cast<int32_t>(row0));
            bulk_commit();
          }
        }
        // both staging blocks read before the dequant warps reuse the region
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
      }
      // no warp writes the next item's weight tiles into a region another warp
      // may still be staging from: every warp arrives, then waits (bounded) for all
      __syncwarp();
      if (lane == 0) mbar_arrive(staging_free);
      if (!__all_sync(0xffffffffu, mbar_wait(staging_free, it & 1, p.status, kFlagTimeoutEpilogue))) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tmem_empty_lead);
    }
  }

  // every output store of this thread has completed
  if (warp >= 2 && lane == 0) bulk_wait<0>();
  // Both CTAs are done with TMEM (the even CTA's MMAs have all completed: every
  // epilogue waited for the last commit or gave up) before the pair frees it.
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
  // Every thread of the owner has consumed the counters by now: clear them for
  // the next launch (nothing else touches them in this one).
  if (threadIdx.x == 64)
    for (int c = (blockIdx.x >> 1) + 1; c < owned_end; ++c) p.counters[2 * c + rank] = 0;
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// Row-major matrix (rows x cols elements of `esize` bytes) -> 2-D tensor map with
// a (box_cols x box_rows) box; box_cols * esize must not exceed the swizzle span.
bool make_map_t(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_cols, int box_rows,
                CUtensorMapDataType dtype, int esize, CUtensorMapSwizzle swizzle) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * esize)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult rc = enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS;
}

// bf16 matrix, 128-byte swizzle (box_cols <= 64).
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_cols, int box_rows) {
  return make_map_t(m, base, rows, cols, box_cols, box_rows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

// ---------------------------------------------------------------- schedule

constexpr int kMinSplitSteps = 16;    // shortest share of the split region per pair (K-steps)
// What one more work item costs a pair, in K-steps of MMA time: the epilogue
// drains the accumulator and the dequant warps refill the pipeline while the MMAs
// wait (5-7 us measured, at about 0.7 us per K-step).
constexpr int kItemCostSteps = 10;
int g_ctas_override = 0;              // qlora_gemm_set_ctas (0: as many pairs as fit)

struct GemmPlan {
  int pairs, tiles_n, dp_tiles, sk_tiles;
};

template <bool kDX, bool kInt>
cudaError_t prepare_kernel() {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && attr_set[dev]) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(nf4_gemm_kernel<kDX, kInt>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemBytes));
  if (e == cudaSuccess && dev >= 0 && dev < 64) attr_set[dev] = true;
  return e;
}

// Pairs (clusters of 2) the device holds at once: every pair of a launch must be
// resident together, since an owner pair may wait for the partials of others.
int device_pairs() {
  static int pairs[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 1;
  }
  if (!pairs[dev]) {
    int n = 0;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (prepare_kernel<false, false>() != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, nf4_gemm_kernel<false, false>, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      return 1;
    }
    pairs[dev] = n;
  }
  return pairs[dev];
}

// Whole pair tiles in full waves; the tiles of the last, partial wave (with one
// more full wave when that alone would give each pair less than half a tile)
// are split evenly by K-steps.  A split region too small for every pair to get
// kMinSplitSteps steps uses fewer pairs, or no split at all.
GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int r, bool split_allowed) {
  const int S = static_cast<int>(K / kBK) + (r + kBK - 1) / kBK;
  const int tiles_n = static_cast<int>((N + kBN - 1) / kBN);
  const int T = tiles_n * static_cast<int>((M + kPairM - 1) / kPairM);
  int C = device_pairs();
  if (g_ctas_override > 0) C = std::min(C, std::max(1, g_ctas_override / 2));
  C = std::min(C, kMaxGemmCtas / 2);
  const GemmPlan whole{std::min(T, C), tiles_n, T, 0};
  if (!split_allowed || T % C == 0) return whole;
  const int waves = T / C, rest = T % C;
  if (waves == 0) {
    // Fewer tiles than pairs: split them only if the shorter range per pair more
    // than pays for the extra work item each pair then runs.
    if (static_cast<int64_t>(T) * S / C + kItemCostSteps >= S) return whole;
    const int pairs = static_cast<int>(std::min<int64_t>(C, static_cast<int64_t>(T) * S / kMinSplitSteps));
    if (pairs <= T) return whole;
    return {pairs, tiles_n, 0, T};
  }
  const int sk = 2 * rest >= C ? rest : rest + C;
  if (static_cast<int64_t>(sk) * S < static_cast<int64_t>(C) * kMinSplitSteps) return whole;
  return {C, tiles_n, T - sk, sk};
}

size_t plan_ws_bytes(const GemmPlan& P) {
  return P.sk_tiles > 0 ? static_cast<size_t>(2 * P.pairs) * kSlotFloats * 4 : 0;
}

template <bool kDX, bool kInt>
cudaError_t launch_gemm(const CUtensorMap& act, const CUtensorMap& ea, const CUtensorMap& eb, const CUtensorMap& cm,
                        const CUtensorMap& om, GemmArgs a, uint32_t* counters, void* partials, size_t partial_bytes,
                        cudaStream_t stream) {
  const cudaError_t pe = prepare_kernel<kDX, kInt>();
  if (pe != cudaSuccess) return pe;
  GemmPlan P = plan_gemm(a.M, a.N, a.K, a.r, partials != nullptr && counters != nullptr);
  if (P.sk_tiles > 0 && partial_bytes < plan_ws_bytes(P)) P = plan_gemm(a.M, a.N, a.K, a.r, false);
  a.tiles_n = P.tiles_n;
  a.dp_tiles = P.dp_tiles;
  a.sk_tiles = P.sk_tiles;
  a.counters = P.sk_tiles > 0 ? counters : nullptr;
  a.partials = P.sk_tiles > 0 ? static_cast<float*>(partials) : nullptr;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * P.pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  const int which = kDX ? QLORA_KERNEL_DX_GEMM : QLORA_KERNEL_FWD_GEMM;
  timing_before(which, stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, nf4_gemm_kernel<kDX, kInt>, act, ea, eb, cm, om, a);
  timing_after(which, stream);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

// Y = X deq(W) + V B.
cudaError_t launch_fwd_gemm(const WeightView& w, const uint16_t* X, const uint16_t* V, const uint16_t* B,
                            int64_t M, int r, uint16_t* Y, uint32_t* status, uint32_t* counters,
                            void* partials, size_t partial_bytes, cudaStream_t stream) {
  CUtensorMap act, ea, eb, cm, om;
  // activations in 128-row boxes; codes as a (in x out/2) byte matrix: 64 rows x
  // 64 bytes (one CTA's 128 columns) per K-step, 64-byte swizzle; Y stored in
  // 32 x 32 blocks, 64-byte swizzle
  if (!make_map(&act, X, M, w.in, 64, 128) || !make_map(&ea, V, M, r, 64, 128) ||
      !make_map(&eb, B, r, w.out, 64, 64) ||
      !make_map_t(&cm, w.codes, w.in, w.out / 2, 64, 64, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_t(&om, Y, M, w.out, 32, 32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  GemmArgs a{w.codes, w.dq_codes, w.dq_scales, w.out, M, w.out, w.in, r, Y, status, w.fmt == kFmtU8 ? 1 : 0,
             0, 0, 0, nullptr, nullptr};
  return w.fmt == kFmtInt16
             ? launch_gemm<false, true>(act, ea, eb, cm, om, a, counters, partials, partial_bytes, stream)
             : launch_gemm<false, false>(act, ea, eb, cm, om, a, counters, partials, partial_bytes, stream);
}

// dX = dY deq(W)^T + U A^T.
cudaError_t launch_dx_gemm(const WeightView& w, const uint16_t* dY, const uint16_t* U, const uint16_t* A,
                           int64_t M, int r, uint16_t* dX, uint32_t* status, uint32_t* counters,
                           void* partials, size_t partial_bytes, cudaStream_t stream) {
  CUtensorMap act, ea, eb, cm, om;
  // activations in 128-row boxes; codes as a (in x out/2) byte matrix: 128 rows
  // (one CTA's columns of dX) x 32 bytes per K-step, 32-byte swizzle; dX stored
  // in 32 x 32 blocks, 64-byte swizzle
  if (!make_map(&act, dY, M, w.out, 64, 128) || !make_map(&ea, U, M, r, 64, 128) ||
      !make_map(&eb, A, w.in, r, 64, 128) ||
      !make_map_t(&cm, w.codes, w.in, w.out / 2, 32, 128, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, CU_TENSOR_MAP_SWIZZLE_32B) ||
      !make_map_t(&om, dX, M, w.in, 32, 32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  GemmArgs a{w.codes, w.dq_codes, w.dq_scales, w.out, M, w.in, w.out, r, dX, status, w.fmt == kFmtU8 ? 1 : 0,
             0, 0, 0, nullptr, nullptr};
  return w.fmt == kFmtInt16
             ? launch_gemm<true, true>(act, ea, eb, cm, om, a, counters, partials, partial_bytes, stream)
             : launch_gemm<true, false>(act, ea, eb, cm, om, a, counters, partials, partial_bytes, stream);
}

size_t fwd_gemm_split_bytes(int64_t M, int64_t n_in, int64_t n_out, int r) {
  return plan_ws_bytes(plan_gemm(M, n_out, n_in, r, true));
}

size_t dx_gemm_split_bytes(int64_t M, int64_t n_in, int64_t n_out, int r) {
  return plan_ws_bytes(plan_gemm(M, n_in, n_out, r, true));
}

void set_gemm_ctas(int ctas) { g_ctas_override = ctas; }

}  // namespace qlora
