// Masked GQA flash attention for sm_100a: TMA-fed K/V staging, tcgen05 MMAs accumulating
// in tensor memory, per-row online softmax, GQA head packing and per-tile mask skipping.
//
// What it computes (sources named by page title and section):
//   out[i, h] = sum_{j < lim(i)} softmax_j(q'[i,h] . k'[j,h/4] * scale) v[j,h/4]
// with 32 query heads over 8 KV heads at head_dim 128 ("hidream-o1-p100a" model card, "What
// this model is"), and lim(i) the exclusive key limit that the HiDream-O1 mask (model card,
// "What this model is"; "HiDream-O1-Image" summary, "How it works") or the HunyuanImage 3.0
// Generalized Causal Attention (paper-graph-ui summary, section 3.4, "The core rule")
// gives row i. Every visible set is a prefix of the keys, so a tile of (query block, key
// block) is either fully visible, fully masked (skipped: no MMA is issued) or needs one
// integer compare per score.
//
// CTA organisation (one CTA per SM, persistent over a longest-first work list):
//   work item = one KV head g, its 4 query heads, 64 consecutive query tokens.
//   The item is two MMA tiles of M = 128 rows; row r of tile X is token
//   q0 + 32 X + r / 4 and query head 4 g + r % 4, so every K/V tile staged in shared
//   memory serves all 4 query heads of its KV head (GQA sharing) and both tiles.
//   warp 0      TMA producer: Q tiles, then K_j, V_j into a 4-slot ring (32 KB per slot)
//   warp 1      TMEM allocator and the single-thread tcgen05.mma issuer
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1 (one thread per row)
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512);
// P (bf16) is written over the first 64 columns of its S and read by the PV MMA from
// tensor memory. The MMA warp interleaves the tiles so that one tile's softmax runs while
// the tensor core works on the other's QK^T and PV:
//   S0(0) S1(0) | PV0(j-1) S0(j) PV1(j-1) S1(j) | ... | PV0(n-1) PV1(n-1)
// A softmax warp publishes P in two halves (keys 0..63, then 64..127), and the MMA warp
// issues the PV MMAs of the first half while the second half is being exponentiated: a
// key block's period is set by each tile's chain S -> softmax -> P -> PV -> S, so work
// moved off that chain is time saved.
// Online softmax keeps the running maximum that was last used for exponentiation and only
// rescales O (in tensor memory) and the row sum when the maximum grows by more than 2^8,
// so probabilities stay below 256 and O is rarely touched.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "exp2_poly.h"
#include "kernels.h"
#include "sm100.cuh"
#include "waits.cuh"

namespace hgx {

namespace {

using namespace sm100;
using namespace waits;

#ifndef HGX_SOFTMAX_SPLIT
#define HGX_SOFTMAX_SPLIT 1
#endif
// Softmax warps per row of a tile: 1 -- one thread holds a whole 128-column row; 2 -- two
// warps on the same tensor-memory lanes each take 64 columns (twice the softmax warps,
// half the dependent work per warp; the row maximum is exchanged through shared memory).
// Both give the same results within rounding; on B200 split 2 measured no faster (the
// exponentials of a row stay on the same SM sub-partition, whose MUFU and issue slots
// they share), so 1 is the default.
constexpr int kSplit = HGX_SOFTMAX_SPLIT;
static_assert(kSplit == 1 || kSplit == 2, "softmax split");
constexpr int kCols = 128 / kSplit;               // score columns per softmax thread
constexpr int kSoftmaxThreads = 128 * kSplit;     // per tile
constexpr int kThreads = 128 + 2 * kSoftmaxThreads;
// register budgets after setmaxnreg (launch: 384 x 168 or 640 x 96 registers)
constexpr uint32_t kRegsLow = kSplit == 1 ? 120 : 64;   // producer/MMA warpgroup
constexpr uint32_t kRegsHigh = kSplit == 1 ? 192 : 104;  // softmax warpgroups
// One Q buffer (both Q tiles of an item): a second one, to load the next item's Q during
// the current item, leaves room for 3 K/V slots only and measured slower.
constexpr int kQBufs = 1;
#ifndef HGX_KV_STAGES
#define HGX_KV_STAGES 4
#endif
constexpr int kStages = HGX_KV_STAGES;        // K/V ring slots
#ifndef HGX_P_PARTS
#define HGX_P_PARTS 2
#endif
// P of a tile is published in this many parts of 128 / kPParts keys (one warp per row), so
// that the PV MMAs of the first parts overlap the exponentials of the later ones
constexpr int kPParts = HGX_P_PARTS;
static_assert(kPParts == 1 || kPParts == 2 || kPParts == 4, "P parts");
#ifndef HGX_SPLIT_LD
#define HGX_SPLIT_LD 1
#endif
// 1: in fully visible blocks the softmax loads S in two halves and takes the maximum of the
// first half while the second half is loading
constexpr bool kSplitLd = HGX_SPLIT_LD != 0 && kSplit == 1;
constexpr uint32_t kTileBytes = 32768;        // 128 rows x 128 bf16
constexpr uint32_t kHalfBytes = 16384;        // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr uint32_t kQBytes = 2 * kTileBytes;  // both Q tiles of an item
constexpr uint32_t kRingOffset = kQBufs * kQBytes;
constexpr uint32_t kBarOffset = kRingOffset + kStages * kTileBytes;
// barrier slots (8 bytes each)
enum : uint32_t {
  BAR_Q_FULL = 0,                    // + Q buffer
  BAR_Q_EMPTY = BAR_Q_FULL + kQBufs, // + Q buffer
  BAR_KV_FULL = BAR_Q_EMPTY + kQBufs,  // + slot
  BAR_KV_EMPTY = BAR_KV_FULL + kStages,
  BAR_S_FULL = BAR_KV_EMPTY + kStages,  // + tile
  BAR_PA_FULL = BAR_S_FULL + 2,         // + tile * (kPParts - 1) + part: that part of P written
  BAR_P_FULL = BAR_PA_FULL + 2 * (kPParts - 1),  // + tile: the last part of P written
  BAR_O_FULL = BAR_P_FULL + 2,
  BAR_O_EMPTY = BAR_O_FULL + 2,
  BAR_STALL = BAR_O_EMPTY + 2,       // debug: nothing ever arrives here
  BAR_DRAIN = BAR_STALL + 1,
  BAR_COUNT = BAR_DRAIN + 1
};
constexpr uint32_t kMiscOffset = kBarOffset + 8 * BAR_COUNT;  // tmem base, abort flag
// row-maximum / row-sum exchange between the two halves of a row (kSplit == 2):
// [iteration parity][tile][half][row] floats
constexpr uint32_t kXchgOffset = kMiscOffset + 16;
constexpr uint32_t kXchgBytes = kSplit == 2 ? 2 * 2 * 2 * 128 * 4 : 0;
#ifndef HGX_EPI_TMA
#define HGX_EPI_TMA 1
#endif
// 1: the epilogue writes O through shared memory with TMA tensor stores: each softmax warp
// stages its 8 tokens x 4 heads x 64 features (4 KB, 128-byte swizzle) and one lane stores
// the box, so that global memory sees whole lines (a warp's direct 16-byte stores touch 32
// rows 256 B apart). Warps with a row outside the element's written range store directly.
constexpr bool kEpiTma = HGX_EPI_TMA != 0 && kSplit == 1;
constexpr uint32_t kEpiOffset = (kXchgOffset + kXchgBytes + 1023u) & ~1023u;
constexpr uint32_t kEpiBytes = kEpiTma ? 8 * 4096 : 0;  // one 4 KB box per softmax warp
constexpr uint32_t kSmemUsed = kEpiOffset + kEpiBytes;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // slack to align the base to 1024 B
static_assert(kSmemBytes <= 232448, "more dynamic shared memory than an sm_100 CTA may have");

constexpr uint32_t kTmemCols = 512;
__host__ __device__ constexpr uint32_t col_s(int x) { return 128u * x; }        // S0, S1
__host__ __device__ constexpr uint32_t col_o(int x) { return 256u + 128u * x; } // O0, O1

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false);  // S = Q K^T, both K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, true);   // O += P V, V N-major

// error sites (bits 8..15 of the error word) to tell which wait ran out
enum : uint32_t {
  SITE_PRODUCER = 1,
  SITE_MMA = 2,
  SITE_SOFTMAX = 3,
  SITE_STALL = 4,
  SITE_DRAIN = 5
};

// S_X = Q_X K^T over head_dim 128: 8 MMAs of K = 16. Both operands K-major with 128-byte
// swizzle: rows of 128 B (64 features), 8-row groups 1024 B apart (SBO); features 64..127
// sit in the second 16 KB half of the tile. The tiles' descriptors are passed in: MMA k
// reads (k >> 2) * 16 KB + (k & 3) * 32 B further on, which adds that offset >> 4 to the
// descriptor's 14-bit start-address field (shared addresses stay below 256 KB, so the
// field never carries into the next one).
__device__ __forceinline__ void issue_qk(uint32_t tmem_s, uint64_t q_desc, uint64_t k_desc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
    mma_ss(tmem_s, q_desc + off, k_desc + off, kIdescQK, kk > 0 ? 1u : 0u);
  }
}

// O_X (+)= P_X V: 8 MMAs of K = 16 keys. P (bf16, 2 per column) is read from tensor
// memory; V is [keys, head_dim] with head_dim contiguous (N-major for the B operand):
// 8-key groups 1024 B apart (SBO), the two 64-feature halves 16 KB apart (LBO).
// MMA k reads keys 16k.. of V, 2 KB further on (descriptor passed in, as for issue_qk).
template <int kFrom, int kTo>  // MMAs kFrom .. kTo - 1: keys 16 * kFrom .. 16 * kTo - 1
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint64_t v_desc,
                                         bool accumulate) {
#pragma unroll
  for (int kk = kFrom; kk < kTo; ++kk)
    mma_ts(tmem_o, tmem_p + kk * 8, v_desc + kk * (2048 >> 4), kIdescPV,
           (accumulate || kk > 0) ? 1u : 0u);
}

#ifndef HGX_EXP_POLY_MASK
// Bit e set: key pair e of every 16 takes the FMA-pipe polynomial exp2 instead of the MUFU
// ex2 (fully visible blocks only). 0 = never.
#define HGX_EXP_POLY_MASK 0
#endif
constexpr bool kExpPolyOn = HGX_EXP_POLY_MASK != 0;

// p = 2^(s * scale_log2 - mb) for scores [kFrom, kTo) of the row's N, packed to bf16 pairs
// and stored as P over the first N/2 columns of S (key 2c in the low half of column c).
// Scale-and-shift and the row sum run as paired fp32 instructions; the row sum is added to
// two pair accumulators.
template <bool kPoly, int N, int kFrom, int kTo>
__device__ __forceinline__ void exp_store_p(const float (&s)[N], float sl2, float mb,
                                            uint32_t tS, uint64_t (&acc)[2]) {
  const uint64_t scale2 = f2_pack(sl2, sl2);
  const uint64_t shift2 = f2_pack(-mb, -mb);
#pragma unroll
  for (int q4 = kFrom / 32; q4 < kTo / 32; ++q4) {  // 32 keys -> 16 packed columns at a time
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float x0, x1;
      f2_unpack(ffma2(f2_pack(s[32 * q4 + 2 * e], s[32 * q4 + 2 * e + 1]), scale2, shift2), x0, x1);
      float p0, p1;
      if (kPoly && ((HGX_EXP_POLY_MASK >> e) & 1)) {
        exp2_poly3_pair(x0, x1, p0, p1);
      } else {
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
      }
      acc[e & 1] = fadd2(acc[e & 1], f2_pack(p0, p1));
      pk[e] = pack_bf16x2(p0, p1);
    }
    tmem_st16(tS + 16 * q4, pk);
  }
}

// The CTA's items: a contiguous list from the host's assignment, or a grid-stride walk.
__device__ __forceinline__ int first_item(const AttnParams& p) {
  return p.cta_offsets ? p.cta_offsets[blockIdx.x] : static_cast<int>(blockIdx.x);
}
__device__ __forceinline__ int end_item(const AttnParams& p) {
  return p.cta_offsets ? p.cta_offsets[blockIdx.x + 1] : p.n_items;
}
__device__ __forceinline__ int next_item(const AttnParams& p, int w) {
  return p.cta_offsets ? w + 1 : w + static_cast<int>(gridDim.x);
}

__global__ void __launch_bounds__(kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v,
                     const __grid_constant__ CUtensorMap tmap_out, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // 128-byte swizzle wants 1024-B alignment
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base;
  const uint32_t sRing = base + kRingOffset;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(gbase + kMiscOffset);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + kMiscOffset + 4);
  Ctx c{base + kBarOffset, abort_flag, p.err, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    for (int b = 0; b < kQBufs; ++b) {
      mbar_init(bar_addr(c, BAR_Q_FULL + b), 1);
      mbar_init(bar_addr(c, BAR_Q_EMPTY + b), 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_addr(c, BAR_KV_FULL + s), 1);
      mbar_init(bar_addr(c, BAR_KV_EMPTY + s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_addr(c, BAR_S_FULL + x), 1);
      for (int i = 0; i < kPParts - 1; ++i)
        mbar_init(bar_addr(c, BAR_PA_FULL + x * (kPParts - 1) + i), kSoftmaxThreads);
      mbar_init(bar_addr(c, BAR_P_FULL + x), kSoftmaxThreads);
      mbar_init(bar_addr(c, BAR_O_FULL + x), 1);
      mbar_init(bar_addr(c, BAR_O_EMPTY + x), kSoftmaxThreads);
    }
    mbar_init(bar_addr(c, BAR_STALL), 1);
    mbar_init(bar_addr(c, BAR_DRAIN), 1);
    *abort_flag = 0u;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_holder)), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (p.stamps && threadIdx.x == 0) {
    p.stamps[4 * blockIdx.x] = clock64();
    p.stamps[4 * blockIdx.x + 1] = globaltimer_ns();
  }

  // Registers (one warp per row): launched at 168 per thread (384 x 168 = 64512). The
  // producer/MMA warpgroup hands registers to the two softmax warpgroups: 128 x 120 +
  // 256 x 192 = 64512, the split at which neither side spills. (Two warps per row: 640
  // threads at 96 registers each, no hand-over.) Only that warpgroup releases and only the softmax
  // warpgroups take, exactly the same amount, so no increase can wait on a warp that is
  // itself waiting; no budget is ever restored (a warp that took back registers early
  // could starve a softmax warp's increase for good). Each role ends in its own branch
  // at a named barrier over all threads, so no code runs under two budgets, and the waits
  // are inlined (a called function cannot serve regions with different budgets).
  if (warp < 4) {
    if constexpr (kRegsLow != kRegsHigh) regs_decrease<kRegsLow>();
    if (warp == 0) {
      // ------------------------------------------------------------------ TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
        uint32_t pos = 0, q_loads = 0;
        uint32_t loaded = 0, last_par = 0;  // per slot: ever loaded, parity of its last load
        bool ok = true;
        // K_j then V_j of block j of an item into the next two ring slots
        auto load_kv = [&](const WorkItem& it, int j) {
          for (int kv = 0; ok && kv < 2; ++kv) {
            const uint32_t slot = pos % kStages;
            const uint32_t round = pos / kStages;
            ok = wait_bounded(c, bar_addr(c, BAR_KV_EMPTY + slot), (round & 1u) ^ 1u, SITE_PRODUCER);
            if (!ok) break;
            const uint32_t full = bar_addr(c, BAR_KV_FULL + slot);
            mbar_arrive_expect_tx(full, kTileBytes);
            const CUtensorMap* map = kv == 0 ? &tmap_k : &tmap_v;
            const int32_t kb =
                it.list_off < 0 ? it.kb0 + j : static_cast<int32_t>(p.kblocks[it.list_off + j] & kListBlockMask);
            for (int hf = 0; hf < 2; ++hf)
              tma_load_3d(sRing + slot * kTileBytes + hf * kHalfBytes, map, full, 64 * hf, it.g,
                          it.kv0 + 128 * kb);
            loaded |= 1u << slot;
            last_par = (last_par & ~(1u << slot)) | ((round & 1u) << slot);
            ++pos;
          }
        };
        for (int w = first_item(p); ok && w < end_item(p); w = next_item(p, w)) {
          const WorkItem it = p.items[w];
          const uint32_t qb = q_loads % kQBufs;  // Q buffer of this item
          if (q_loads >= static_cast<uint32_t>(kQBufs)) {
            ok = wait_bounded(c, bar_addr(c, BAR_Q_EMPTY + qb), ((q_loads / kQBufs) - 1) & 1u, SITE_PRODUCER);
            if (!ok) break;
          }
          mbar_arrive_expect_tx(bar_addr(c, BAR_Q_FULL + qb), kQBytes);
          for (int x = 0; x < 2; ++x) {
            // a tile that starts past the last token only holds rows that are never stored:
            // start it at the last token so that no box lies wholly outside the tensor
            const int32_t t0 = min(it.q0 + 32 * x, p.total_tokens - 1);
            for (int hf = 0; hf < 2; ++hf)
              tma_load_3d(sQ + qb * kQBytes + x * kTileBytes + hf * kHalfBytes, &tmap_q, bar_addr(c, BAR_Q_FULL + qb),
                          64 * hf, 4 * it.g, t0);
          }
          ++q_loads;
          for (int j = 0; ok && j < it.n_total; ++j) load_kv(it, j);
        }
        // drain: every load this thread issued must land before the CTA exits (on the normal
        // path they all have, and these waits return at once)
        for (int s = 0; s < kStages; ++s)
          if (loaded & (1u << s)) wait_drain(c, bar_addr(c, BAR_KV_FULL + s), (last_par >> s) & 1u, SITE_DRAIN);
        for (uint32_t b = 0; b < static_cast<uint32_t>(kQBufs) && b < q_loads; ++b) {  // last load of buffer b
          const uint32_t last = q_loads - 1 - ((q_loads - 1 - b) % kQBufs);
          wait_drain(c, bar_addr(c, BAR_Q_FULL + b), (last / kQBufs) & 1u, SITE_DRAIN);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        uint32_t pos = 0, q_items = 0;
        uint32_t pa_par[2] = {0, 0}, p_par[2] = {0, 0}, oe_par[2] = {0, 0};  // pa: all parts share it
        bool first = true, ok = true;
        auto wait_kv = [&](uint32_t ps) {
          return wait_bounded(c, bar_addr(c, BAR_KV_FULL + ps % kStages), (ps / kStages) & 1u,
                              SITE_MMA);
        };
        // descriptors of both Q tiles and of K / V in ring slot 0 (slot s: + s * 32 KB >> 4)
        const uint64_t dq0_base = smem_desc_sw128(sQ, 16, 1024);
        const uint64_t dq1_base = smem_desc_sw128(sQ + kTileBytes, 16, 1024);
        const uint64_t dk0 = smem_desc_sw128(sRing, 16, 1024);
        const uint64_t dv0 = smem_desc_sw128(sRing, kHalfBytes, 1024);
        auto kdesc = [&](uint32_t ps) { return dk0 + (ps % kStages) * (kTileBytes >> 4); };
        auto vdesc = [&](uint32_t ps) { return dv0 + (ps % kStages) * (kTileBytes >> 4); };
        auto release = [&](uint32_t ps) { mma_commit(bar_addr(c, BAR_KV_EMPTY + ps % kStages)); };
        // wait until softmax X has written part `part` of P (the first part: and rescaled O);
        // before the first PV of an item also wait until the previous item's epilogue has
        // read O. The parts other than the last have barriers of their own, which all
        // complete once per block, so they share one parity.
        auto wait_part = [&](int x, int part, bool first_pv) {
          const bool last = part == kPParts - 1;
          const uint32_t bar = last ? BAR_P_FULL + x : BAR_PA_FULL + x * (kPParts - 1) + part;
          if (!wait_bounded(c, bar_addr(c, bar), last ? p_par[x] : pa_par[x], SITE_MMA)) return false;
          if (last) p_par[x] ^= 1u;
          else if (part == kPParts - 2) pa_par[x] ^= 1u;
          if (part == 0 && first_pv && !first) {
            if (!wait_bounded(c, bar_addr(c, BAR_O_EMPTY + x), oe_par[x], SITE_MMA)) return false;
            oe_par[x] ^= 1u;
          }
          tc_fence_after();
          return true;
        };
        // O_X (+)= P_X V in kPParts parts, each issued as soon as its part of P is in tensor
        // memory: the first parts run while the softmax exponentiates the later ones
        auto pv = [&](int x, uint32_t ps, bool accumulate, bool first_pv) {
          constexpr int kStep = 8 / kPParts;
          if (!wait_part(x, 0, first_pv)) return false;
          issue_pv<0, kStep>(tmem + col_o(x), tmem + col_s(x), vdesc(ps), accumulate);
          if constexpr (kPParts >= 2) {
            if (!wait_part(x, 1, first_pv)) return false;
            issue_pv<kStep, 2 * kStep>(tmem + col_o(x), tmem + col_s(x), vdesc(ps), accumulate);
          }
          if constexpr (kPParts == 4) {
            if (!wait_part(x, 2, first_pv)) return false;
            issue_pv<2 * kStep, 3 * kStep>(tmem + col_o(x), tmem + col_s(x), vdesc(ps), accumulate);
            if (!wait_part(x, 3, first_pv)) return false;
            issue_pv<3 * kStep, 4 * kStep>(tmem + col_o(x), tmem + col_s(x), vdesc(ps), accumulate);
          }
          return true;
        };
        for (int w = first_item(p); ok && w < end_item(p); w = next_item(p, w)) {
          const WorkItem it = p.items[w];
          const int n = it.n_total;
          const uint32_t qb = q_items % kQBufs;
          if (!(ok = wait_bounded(c, bar_addr(c, BAR_Q_FULL + qb), (q_items / kQBufs) & 1u, SITE_MMA))) break;
          ++q_items;
          const uint64_t dq0 = dq0_base + qb * (kQBytes >> 4), dq1 = dq1_base + qb * (kQBytes >> 4);
          uint32_t kpos = pos++;
          if (!(ok = wait_kv(kpos))) break;
          tc_fence_after();
          issue_qk(tmem + col_s(0), dq0, kdesc(kpos));
          mma_commit(bar_addr(c, BAR_S_FULL + 0));
          issue_qk(tmem + col_s(1), dq1, kdesc(kpos));
          mma_commit(bar_addr(c, BAR_S_FULL + 1));
          if (n == 1) mma_commit(bar_addr(c, BAR_Q_EMPTY + qb));
          release(kpos);
          for (int j = 1; j < n; ++j) {
            const uint32_t vpos = pos++;
            kpos = pos++;
            if (!(ok = wait_kv(vpos) && wait_kv(kpos))) break;
            if (!(ok = pv(0, vpos, j > 1, j == 1))) break;
            issue_qk(tmem + col_s(0), dq0, kdesc(kpos));
            mma_commit(bar_addr(c, BAR_S_FULL + 0));
            if (!(ok = pv(1, vpos, j > 1, j == 1))) break;
            release(vpos);
            issue_qk(tmem + col_s(1), dq1, kdesc(kpos));
            mma_commit(bar_addr(c, BAR_S_FULL + 1));
            if (j == n - 1) mma_commit(bar_addr(c, BAR_Q_EMPTY + qb));
            release(kpos);
          }
          if (!ok) break;
          const uint32_t vpos = pos++;
          if (!(ok = wait_kv(vpos))) break;
          if (!(ok = pv(0, vpos, n > 1, n == 1))) break;
          mma_commit(bar_addr(c, BAR_O_FULL + 0));
          if (!(ok = pv(1, vpos, n > 1, n == 1))) break;
          mma_commit(bar_addr(c, BAR_O_FULL + 1));
          release(vpos);
          first = false;
        }
        // every MMA this thread issued must complete before tensor memory is freed
        mma_commit(bar_addr(c, BAR_DRAIN));
        wait_drain(c, bar_addr(c, BAR_DRAIN), 0, SITE_DRAIN);
      }
      __syncwarp();
    }
    // end of the producer/MMA warpgroup: wait for every role, then free tensor memory
    tc_fence_before();
    named_bar_sync(1, kThreads);
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
    if (p.stamps && threadIdx.x == 0) {  // every role of the CTA has passed the barrier
      p.stamps[4 * blockIdx.x + 2] = clock64();
      p.stamps[4 * blockIdx.x + 3] = globaltimer_ns();
    }
  } else {
    if constexpr (kRegsLow != kRegsHigh) regs_increase<kRegsHigh>();
    // ------------------------------------------------------------------ softmax
    const int x = (warp - 4) / (4 * kSplit);     // tile
    const int half = ((warp - 4) >> 2) % kSplit;  // which kCols columns of the row
    const int quarter = warp & 3;                // tensor-memory lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_bits + col_s(x) + kCols * half;      // S columns
    const uint32_t tP = tmem + lane_bits + col_s(x) + kCols / 2 * half;  // P columns
    const uint32_t tO = tmem + lane_bits + col_o(x) + kCols * half;      // O columns
    float* xchg = reinterpret_cast<float*>(gbase + kXchgOffset);
    const float sl2 = p.scale_log2;
    uint32_t s_par = 0, o_par = 0;
    int xpar = 0;  // exchange buffer parity
    uint32_t ring = 0;        // K/V ring position of the next key block's K (V follows it)
    uint8_t* const ring_g = gbase + kRingOffset;
    // one decision for every thread of the tile: its two halves must leave together
    auto agree = [&](bool v) {
      if constexpr (kSplit == 1) return __all_sync(0xffffffffu, v);
      else return named_bar_and(2 + x, kSoftmaxThreads, v);
    };
    bool ok = true;
    if ((p.flags & HGX_DEBUG_STALL_TEST) && x == 0)
      ok = agree(wait_bounded(c, bar_addr(c, BAR_STALL), 0, SITE_STALL));
    for (int w = first_item(p); ok && w < end_item(p); w = next_item(p, w)) {
      const WorkItem it = p.items[w];
      const int32_t tok = it.q0 + 32 * x + (row >> 2);
      const int32_t head = 4 * it.g + (row & 3);
      const bool valid = tok - it.kv0 < it.len && tok - it.kv0 >= it.first;
      const int32_t row_lim = valid ? p.lim[tok] : it.len;
      const bool listed = it.list_off >= 0;  // item whose rows see a Gen Image hole
      const int32_t hbase = (listed && valid) ? p.hole_base[tok] : -1;
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < it.n_total; ++j) {
        // key block and its class (read before the wait, which hides the load)
        const uint32_t entry = listed ? p.kblocks[it.list_off + j] : 0u;
        const int32_t kb = listed ? static_cast<int32_t>(entry & kListBlockMask) : it.kb0 + j;
        const bool full = listed ? (entry >> kListClassShift) == HGX_TILE_FULL : kb < it.n_full;
        uint4 hm = make_uint4(0u, 0u, 0u, 0u);
        if (!full && hbase >= 0)
          hm = *reinterpret_cast<const uint4*>(p.hole_masks + 4 * static_cast<size_t>(hbase + kb));
        bool got = wait_bounded(c, bar_addr(c, BAR_S_FULL + x), s_par, SITE_SOFTMAX);
        const uint32_t vpos = ring + 1;
        ring += 2;
        // A key block that runs past the end of its batch element into the next one: the
        // probabilities of those keys are exact zeros, but their V rows belong to the next
        // element and 0 * inf or 0 * NaN would be NaN, so tile 0 zeroes them in shared
        // memory once the V tile has landed and before it publishes any P of this block
        // (the PV MMAs of both tiles read V after that). Blocks past the last token read
        // zeros from the tensor map already.
        if (x == 0 && 128 * kb + 128 > it.len && it.kv0 + it.len < p.total_tokens) {
          got = got && wait_bounded(c, bar_addr(c, BAR_KV_FULL + vpos % kStages), (vpos / kStages) & 1u,
                                    SITE_SOFTMAX);
          if (half == 0 && row >= it.len - 128 * kb) {
            uint8_t* v_row = ring_g + (vpos % kStages) * kTileBytes + row * 128;
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
              for (int e = 0; e < 8; ++e) reinterpret_cast<uint4*>(v_row + hf * kHalfBytes)[e] = z;
          }
          fence_proxy_async_smem();  // the tensor core reads these rows through the async proxy
        }
        if constexpr (kSplit == 1) {
          if (!(ok = __all_sync(0xffffffffu, got))) break;
        }
        s_par ^= 1u;
        tc_fence_after();
        // (with two halves an aborted wait still loads: tensor memory is always readable,
        // and the tile decides together at the exchange below)
        uint32_t sr[kCols / 32][32];
        float s[kCols];
        float mx;
        // row max: independent chains of 16 scores (three-input max), then a tree; a single
        // long chain would expose its whole latency
        auto chain16 = [&](int i) {
          const float* c16 = s + 16 * i;
          float m = fmax3(c16[0], c16[1], c16[2]);
#pragma unroll
          for (int e = 3; e < 15; e += 2) m = fmax3(m, c16[e], c16[e + 1]);
          return fmaxf(m, c16[15]);
        };
        if (kSplitLd && full) {
          // a fully visible block: the second half of the row loads while the maximum of
          // the first half is computed
          tmem_ld32(tS, sr[0]);
          tmem_ld32(tS + 32, sr[1]);
          tmem_wait_ld();
          tmem_ld32(tS + 64, sr[2]);
          tmem_ld32(tS + 96, sr[3]);
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
#pragma unroll
            for (int e = 0; e < 32; ++e) s[32 * ch + e] = __uint_as_float(sr[ch][e]);
          const float ma = fmaxf(fmaxf(chain16(0), chain16(1)), fmaxf(chain16(2), chain16(3)));
          tmem_wait_ld();
#pragma unroll
          for (int ch = 2; ch < 4; ++ch)
#pragma unroll
            for (int e = 0; e < 32; ++e) s[32 * ch + e] = __uint_as_float(sr[ch][e]);
          mx = fmaxf(ma, fmaxf(fmaxf(chain16(4), chain16(5)), fmaxf(chain16(6), chain16(7))));
        } else {
#pragma unroll
        for (int ch = 0; ch < kCols / 32; ++ch) tmem_ld32(tS + 32 * ch, sr[ch]);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < kCols / 32; ++ch)
#pragma unroll
          for (int e = 0; e < 32; ++e) s[32 * ch + e] = __uint_as_float(sr[ch][e]);
        if (!full) {
          // keys [0, nvis) of this block are in the prefix
          const int nvis = row_lim - 128 * kb - kCols * half;
          if (hbase >= 0) {
            // keys hidden by Gen Image holes: the mask words of this thread's columns, picked
            // up front so that every index below is a compile-time constant
            uint32_t hw[kCols / 32];
            if constexpr (kSplit == 1) {
              hw[0] = hm.x; hw[1] = hm.y; hw[2 % (kCols / 32)] = hm.z; hw[3 % (kCols / 32)] = hm.w;
            } else {
              hw[0] = half ? hm.z : hm.x;
              hw[1] = half ? hm.w : hm.y;
            }
#pragma unroll
            for (int e = 0; e < kCols; ++e)
              if (e >= nvis || ((hw[e >> 5] >> (e & 31)) & 1u)) s[e] = -INFINITY;
          } else {
#pragma unroll
            for (int e = 0; e < kCols; ++e)
              if (e >= nvis) s[e] = -INFINITY;
          }
        }
        float m8[kCols / 16];
#pragma unroll
        for (int i = 0; i < kCols / 16; ++i) m8[i] = chain16(i);
        mx = m8[0];
#pragma unroll
        for (int i = 1; i < kCols / 16; ++i) mx = fmaxf(mx, m8[i]);
        }
        if constexpr (kSplit == 2) {
          // exchange with the other half of the row; the barrier also decides, for the
          // whole tile, whether every wait succeeded
          float* slot = xchg + ((xpar * 2 + x) * 2) * 128;
          slot[half * 128 + row] = mx;
          // the barrier also orders this half's S loads before the other half's P stores,
          // which overwrite S columns 32..63 of the tile
          tc_fence_before();
          if (!(ok = named_bar_and(2 + x, kSoftmaxThreads, got))) break;
          tc_fence_after();
          mx = fmaxf(mx, slot[(half ^ 1) * 128 + row]);
          xpar ^= 1;
        }
        const float m_new = fmaxf(m_used, mx);
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_used = m_new;
        } else if (__any_sync(0xffffffffu, (m_new - m_used) * sl2 > 8.0f)) {
          // warp-uniform: the tensor-memory loads and stores of the O rescale are
          // warp-collective, so when any row of the warp needs it every row rescales (by
          // its own factor <= 1); both halves of a row see the same maxima, so they agree
          alpha = ex2_approx((m_used - m_new) * sl2);
          m_used = m_new;
          rescale = true;
        }
        // a row whose keys so far were all hidden (a Gen Image hole before its first visible
        // key) still has m_used = -inf: exponentiate against 0, so its masked scores give
        // exact zeros and its first real maximum later rescales the all-zero O by 0
        const float mb = m_used == -INFINITY ? 0.f : m_used * sl2;
        // exponentials and P. With one warp per row, P is written in kPParts parts and each
        // part but the last is published before the next is exponentiated, so that the PV
        // MMAs of the early parts overlap the later exponentials -- unless O must be rescaled
        // first (rare): then every part is published after the rescale.
        uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
        constexpr int kParts = kSplit == 1 ? kPParts : 1;
        constexpr int kW = kCols / kParts;  // keys per part
        const bool early = kParts > 1 && !rescale;
        auto publish = [&](int part) {
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar_addr(c, BAR_PA_FULL + x * (kPParts - 1) + part));
        };
        auto exp_part = [&](auto from_c, auto to_c) {
          constexpr int kFrom = decltype(from_c)::value, kTo = decltype(to_c)::value;
          if (kExpPolyOn && full)
            exp_store_p<true, kCols, kFrom, kTo>(s, sl2, mb, tP, acc);  // no -inf: polynomial allowed
          else
            exp_store_p<false, kCols, kFrom, kTo>(s, sl2, mb, tP, acc);  // MUFU: zeros for -inf
        };
        exp_part(std::integral_constant<int, 0>{}, std::integral_constant<int, kW>{});
        if constexpr (kParts >= 2) {
          if (early) publish(0);
          exp_part(std::integral_constant<int, kW>{}, std::integral_constant<int, 2 * kW>{});
        }
        if constexpr (kParts == 4) {
          if (early) publish(1);
          exp_part(std::integral_constant<int, 2 * kW>{}, std::integral_constant<int, 3 * kW>{});
          if (early) publish(2);
          exp_part(std::integral_constant<int, 3 * kW>{}, std::integral_constant<int, 4 * kW>{});
        }
        float l4[4];
        f2_unpack(acc[0], l4[0], l4[1]);
        f2_unpack(acc[1], l4[2], l4[3]);
        l = fmaf(l, alpha, (l4[0] + l4[1]) + (l4[2] + l4[3]));
        if (rescale) {
          // O may be touched now: the PV of the previous block completed before S of this
          // one (one commit tracks both), and the PVs of this block wait for the P barriers
          // below
#pragma unroll
          for (int ch = 0; ch < kCols / 32; ++ch) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * ch, o);
            tmem_wait_ld();
            const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float lo, hi;
              f2_unpack(fmul2(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2), lo, hi);
              o[e] = __float_as_uint(lo);
              o[e + 1] = __float_as_uint(hi);
            }
            tmem_st32(tO + 32 * ch, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        if (!early)  // every part at once
          for (int i = 0; i < kPParts - 1; ++i) mbar_arrive(bar_addr(c, BAR_PA_FULL + x * (kPParts - 1) + i));
        mbar_arrive(bar_addr(c, BAR_P_FULL + x));
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 -> out[tok, head, :]
      const bool got = wait_bounded(c, bar_addr(c, BAR_O_FULL + x), o_par, SITE_SOFTMAX);
      if constexpr (kSplit == 2) {
        float* slot = xchg + ((xpar * 2 + x) * 2) * 128;
        slot[half * 128 + row] = l;
        ok = named_bar_and(2 + x, kSoftmaxThreads, got);
        if (ok) l += slot[(half ^ 1) * 128 + row];
        xpar ^= 1;
      } else {
        ok = __all_sync(0xffffffffu, got);
      }
      if (!ok) break;
      o_par ^= 1u;
      tc_fence_after();
      if (it.part >= 0) {
        // one part of a split item: unnormalised O, the exponent shift and the row sum, for
        // the combine kernel (a row that saw no key of this part has l = 0 and M = -inf)
        const size_t prow = (static_cast<size_t>(it.part) * 2 + x) * 128 + row;
        float* po = p.partial_o + prow * 128 + kCols * half;
#pragma unroll
        for (int ch = 0; ch < kCols / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * ch, o);
          tmem_wait_ld();
          if (valid) {
            float4* d4 = reinterpret_cast<float4*>(po + 32 * ch);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              d4[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                  __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
          }
        }
        if (valid && half == 0)
          p.partial_ml[prow] = make_float2(m_used == -INFINITY ? -INFINITY : m_used * sl2, l);
        tc_fence_before();
        mbar_arrive(bar_addr(c, BAR_O_EMPTY + x));
        continue;
      }
      const float inv_l = 1.0f / l;
      if (kEpiTma && p.out_tma && __all_sync(0xffffffffu, valid)) {
        // stage this warp's 32 rows = 8 tokens x 4 heads, 64 features at a time, in the
        // 128-byte-swizzled box layout (row = lane, 16-byte chunk j at j ^ (lane & 7)), and
        // store each box with one TMA store
        const uint32_t stage = base + kEpiOffset + ((warp - 4) & 7) * 4096u;
        uint8_t* stage_g = gbase + kEpiOffset + ((warp - 4) & 7) * 4096u;
        const int32_t tok0 = it.q0 + 32 * x + 8 * quarter;
#pragma unroll
        for (int c64 = 0; c64 < 2; ++c64) {
          uint32_t o[2][32];
          tmem_ld32(tO + 64 * c64, o[0]);
          tmem_ld32(tO + 64 * c64 + 32, o[1]);
          tmem_wait_ld();
          // the warp's previous box (the first half, or the last item's second half) must
          // have left shared memory before it is overwritten
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t* w = o[j >> 2] + 8 * (j & 3);
            const uint4 v = make_uint4(pack_bf16x2(__uint_as_float(w[0]) * inv_l, __uint_as_float(w[1]) * inv_l),
                                       pack_bf16x2(__uint_as_float(w[2]) * inv_l, __uint_as_float(w[3]) * inv_l),
                                       pack_bf16x2(__uint_as_float(w[4]) * inv_l, __uint_as_float(w[5]) * inv_l),
                                       pack_bf16x2(__uint_as_float(w[6]) * inv_l, __uint_as_float(w[7]) * inv_l));
            *reinterpret_cast<uint4*>(stage_g + lane * 128 + ((j ^ (lane & 7)) << 4)) = v;
          }
          fence_proxy_async_smem();  // the TMA reads the staged box through the async proxy
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmap_out, stage, 64 * c64, 4 * it.g, tok0);
            bulk_commit_group();
          }
        }
        tc_fence_before();
        mbar_arrive(bar_addr(c, BAR_O_EMPTY + x));
        continue;
      }
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) +
                           (static_cast<size_t>(tok) * 32 + head) * 128 + kCols * half;
#pragma unroll
      for (int ch = 0; ch < kCols / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * ch, o);
        tmem_wait_ld();
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l,
                                __uint_as_float(o[2 * e + 1]) * inv_l);
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * ch);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_addr(c, BAR_O_EMPTY + x));
    }
    if (kEpiTma && lane == 0) bulk_wait_all();  // this warp's box stores have completed
    tc_fence_before();
    named_bar_sync(1, kThreads);  // pairs with the producer/MMA warpgroup's barrier
  }
}

// One warp per row of a split item: out = sum_p O_p 2^(M_p - M) / sum_p l_p 2^(M_p - M),
// M = max M_p over the parts the row saw keys in. Lane i first reads the (M, l) of parts i,
// i + 32, ... (all at once), the warp reduces the maximum and the denominator with
// shuffles, and then every lane accumulates features 4i .. 4i + 3 over the parts with
// independent loads (a part whose row saw no key has O = 0 and weight 0).
__global__ void __launch_bounds__(256) combine_kernel(const WorkItem* __restrict__ splits, int32_t n_splits,
                                                      const float* __restrict__ po,
                                                      const float2* __restrict__ pml, __nv_bfloat16* out) {
  const int32_t gw = static_cast<int32_t>(blockIdx.x) * 8 + static_cast<int32_t>(threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= n_splits * 256) return;
  const WorkItem it = splits[gw >> 8];
  const int x = (gw >> 7) & 1, row = gw & 127;
  const int32_t tok = it.q0 + 32 * x + (row >> 2);
  if (!(tok - it.kv0 < it.len && tok - it.kv0 >= it.first)) return;
  auto prow = [&](int i) { return (static_cast<size_t>(it.part + i) * 2 + x) * 128 + row; };
  const int np = it.n_parts;
  float m = -INFINITY;
  for (int i = lane; i < np; i += 32) {
    const float2 ml = pml[prow(i)];
    if (ml.y > 0.f) m = fmaxf(m, ml.x);  // finite: every written row sees at least itself
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float den = 0.f;
  for (int i = lane; i < np; i += 32) {
    const float2 ml = pml[prow(i)];
    if (ml.y > 0.f) den = fmaf(ml.y, exp2f(ml.x - m), den);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int i = 0; i < np; ++i) {
    const float2 ml = pml[prow(i)];  // the same address for all lanes: one broadcast load
    const float wgt = ml.y > 0.f ? exp2f(ml.x - m) : 0.f;
    const float4 o = reinterpret_cast<const float4*>(po + prow(i) * 128)[lane];
    acc.x = fmaf(o.x, wgt, acc.x);
    acc.y = fmaf(o.y, wgt, acc.y);
    acc.z = fmaf(o.z, wgt, acc.z);
    acc.w = fmaf(o.w, wgt, acc.w);
  }
  const float inv = 1.f / den;
  const uint32_t lo = pack_bf16x2(acc.x * inv, acc.y * inv);
  const uint32_t hi = pack_bf16x2(acc.z * inv, acc.w * inv);
  const int32_t head = 4 * it.g + (row & 3);
  reinterpret_cast<uint2*>(out + (static_cast<size_t>(tok) * 32 + head) * 128)[lane] = make_uint2(lo, hi);
}

}  // namespace

cudaError_t launch_combine(cudaStream_t stream, const WorkItem* splits, int32_t n_splits,
                           const float* partial_o, const float2* partial_ml, void* out) {
  if (n_splits <= 0) return cudaSuccess;
  const int blocks = (n_splits * 256 + 7) / 8;
  combine_kernel<<<blocks, 256, 0, stream>>>(splits, n_splits, partial_o, partial_ml,
                                             static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

size_t attention_smem_bytes() { return kSmemBytes; }

cudaError_t launch_attention(cudaStream_t stream, const CUtensorMap& tmap_q,
                             const CUtensorMap& tmap_k, const CUtensorMap& tmap_v,
                             const CUtensorMap& tmap_out, const AttnParams& p, int grid) {
  static uint64_t configured = 0;  // bit per device: shared-memory limit raised
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    e = cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    if (dev < 64) configured |= 1ull << dev;
  }
  attention_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tmap_q, tmap_k, tmap_v, tmap_out, p);
  return cudaGetLastError();
}

}  // namespace hgx
