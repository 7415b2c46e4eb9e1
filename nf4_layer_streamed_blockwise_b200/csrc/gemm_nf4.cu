// Fused NF4-dequant GEMMs with the LoRA path, sm_100a: tcgen05 on SM pairs.
//
//   FWD: Y = residual + X deq(W)^T + s U B^T,          U = X A^T
//   DX : dX = sum_seg dY_seg deq(W_seg) + s G A,       G = [G_seg] = [dY_seg B_seg]
//
// Main kernel (nf4_pair_kernel<MODE, H>).  A cluster of two CTAs on two SMs
// computes a (256 H) x 256 output tile with tcgen05.mma.cta_group::2 (M = 256,
// N = 256, H instructions per k-step): each CTA stages its own H x 128
// activation rows and decodes its own 128 columns of the weight tile into
// shared memory, and the pair's tensor cores read both halves.  Per SM that is
// half the weight-operand reads and half the decode work per FLOP of a one-SM
// tile, and with H = 2 each decoded weight tile feeds two 128-row halves.  The
// kernel is persistent: cluster c takes tiles c, c + C, c + 2C, ... (C
// clusters, m index fastest so that the clusters in flight share weight
// columns in L2).  H = 1 alternates two TMEM accumulators (the epilogue of one
// tile overlaps the main loop of the next, six stages); H = 2 fills TMEM with
// one 512-column accumulator pair (four stages).  With a stream-K workspace
// the last round or two of tiles are shared out as equal ranges of weight
// blocks (see piece_at and launch_pair).
//
// The rank-r products stay off the main loop: a split-K tcgen05 kernel
// (lora_down_kernel) computes U = X A^T (or G = dY B), reduces its splits
// inside a thread-block cluster and writes U in fp32 and s*U (s*G) in bf16,
// zero-padded to 64 columns.  The main loop then runs (s U) B^T (or (s G) A)
// as one extra contraction block of width 64 whose two operands are
// TMA-loaded like the activation tile, so the output is still rounded to bf16
// once.  A rank state (state_plan) keeps s*U and the padded / transposed
// LoRA operands from a layer's first forward for its checkpoint recompute and
// backward.
//
// Warp roles in each CTA of the pair:
//   0-3   epilogue: TMEM lanes 0-127 -> the CTA's 128 output rows
//   9     TMA producer: activation tile, packed codes, the LoRA block's tiles
//   5     TMEM owner; in the leader CTA (rank 0) also the MMA issuer
//   4, 6-8, 10-12, 14  NF4 decoders: two threads per 64-value block of the
//         stage, each writing half of one 128-byte row of the swizzled bf16
//         operand; the block's 16 possible values live in registers
//         (byte-permute decode, eight codes per step)
//   13    idle: the issuing warps 5 and 9 have SM sub-partition 1 to
//         themselves (see NTHREADS)
// The leader's "full" barrier of a stage completes when both CTAs' TMA bytes
// have landed and all 16 decoder warps of the pair have arrived; the MMA
// commit releases the stage in both CTAs at once (commit multicast).  Every
// wait is bounded (common.cuh); there are no atomics, so results do not
// depend on timing or on which SM ran which tile (stream-K partials are added
// in cluster order).
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdlib>

#include "common.cuh"
#include "host_common.h"

namespace lsq {
namespace nf4g {

enum Mode { FWD = 0, DX = 1 };

// ---------------------------------------------------------------- cluster / CTA-pair PTX
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of this CTA's variable p as seen in CTA `rank`
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Arrive on an mbarrier of either CTA of the pair (default .release.cta
// semantics).  The writes this arrival publishes are shared-memory tiles that
// the tensor cores read through the async proxy: the writer's
// fence.proxy.async orders them, so a cluster-scope release, which costs a
// full memory fence on every arrival, buys nothing here.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
// all threads of both CTAs
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 2-D tile load into this CTA's shared memory that completes on an mbarrier of
// either CTA of the pair (here always the leader's)
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* m, uint32_t bar_caddr, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(m), "r"(bar_caddr), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (+)= A B^T over the pair: A rows 0-127 from the leader's shared memory,
// 128-255 from the peer's; B rows (output columns) split the same way.
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the barrier at this offset in every CTA of `mask` once all MMAs issued so far complete
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t* bar, uint16_t mask) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::
                   "r"(smem_u32(bar)),
               "h"(mask)
               : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// The 16 dequantised values bf16(code_value[c] * absmax) of one NF4 block, held
// in registers as byte planes: lo[j] / hi[j] are the low / high bytes of
// entries 4j .. 4j+3.  Decoding then selects bytes with prmt instead of
// looking the codebook up in shared memory per value: the same fp32 product
// and round-to-nearest-even as lsq_nf4_dequantize, computed once per code
// value and block, and no shared-memory traffic per value.
struct DqTab {
  uint32_t lo[4], hi[4];
};
__device__ __forceinline__ DqTab dq_table(float a, const float (&cb)[16]) {
  DqTab t;
  const uint64_t aa = f2(a, a);  // paired fp32 multiplies: each lane rounded as __fmul_rn
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t t0 = pack_bf16x2(mul2(f2(cb[4 * j], cb[4 * j + 1]), aa));
    const uint32_t t1 = pack_bf16x2(mul2(f2(cb[4 * j + 2], cb[4 * j + 3]), aa));
    t.lo[j] = prmt(t0, t1, 0x6420u);
    t.hi[j] = prmt(t0, t1, 0x7531u);
  }
  return t;
}
// Four codes in the low 16 bits of ch (byte 0 = codes 0 | 1, high nibble
// first) -> four bf16 as two words.  prmt selects one of 8 bytes by the low 3
// bits of a selector nibble, so each plane is read as two 8-entry halves and
// the half is chosen per byte by bit 3 of the code (mask m: 0xFF where set).
__device__ __forceinline__ uint2 dq4(uint32_t ch, const DqTab& t) {
  const uint32_t s7 = ch & 0x7777u, c8 = ch & 0x8888u;
  const uint32_t m = prmt(0u, 0x80u, c8 | (c8 >> 1));  // nibble 0xC: sign of byte 4 (0x80) -> 0xFF; 0 -> 0x00
  const uint32_t lo = (prmt(t.lo[0], t.lo[1], s7) & ~m) | (prmt(t.lo[2], t.lo[3], s7) & m);
  const uint32_t hi = (prmt(t.hi[0], t.hi[1], s7) & ~m) | (prmt(t.hi[2], t.hi[3], s7) & m);
  // lo / hi bytes are ordered (code 1, code 0, code 3, code 2): interleave to bf16 words
  return make_uint2(prmt(lo, hi, 0x4051u), prmt(lo, hi, 0x6273u));
}
// eight codes (one 32-bit word) -> eight bf16: dq4 of the low and the high half-word, with the
// code and sign masks formed once on the whole word (prmt reads only the low 16 bits of its
// selector, and the shifted sign bits stay inside their half-word)
__device__ __forceinline__ uint4 dq8(uint32_t w, const DqTab& t) {
  const uint32_t s7 = w & 0x77777777u, c8 = w & 0x88888888u;
  const uint32_t sel = c8 | (c8 >> 1), s7h = s7 >> 16;
  const uint32_t m0 = prmt(0u, 0x80u, sel), m1 = prmt(0u, 0x80u, sel >> 16);
  const uint32_t lo0 = (prmt(t.lo[0], t.lo[1], s7) & ~m0) | (prmt(t.lo[2], t.lo[3], s7) & m0);
  const uint32_t hi0 = (prmt(t.hi[0], t.hi[1], s7) & ~m0) | (prmt(t.hi[2], t.hi[3], s7) & m0);
  const uint32_t lo1 = (prmt(t.lo[0], t.lo[1], s7h) & ~m1) | (prmt(t.lo[2], t.lo[3], s7h) & m1);
  const uint32_t hi1 = (prmt(t.hi[0], t.hi[1], s7h) & ~m1) | (prmt(t.hi[2], t.hi[3], s7h) & m1);
  return make_uint4(prmt(lo0, hi0, 0x4051u), prmt(lo0, hi0, 0x6273u), prmt(lo1, hi1, 0x4051u),
                    prmt(lo1, hi1, 0x6273u));
}

// half of an NF4 block (32 values, 16 code bytes) -> 16-byte chunks
// half*4 .. half*4+3 of one 128-byte row of a 128B-swizzled tile
__device__ __forceinline__ void store_half_row(uint32_t row_addr, int row, int half, uint4 c, const DqTab& t) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) st_shared_v4(row_addr + ((uint32_t)((half * 4 + q) ^ (row & 7)) << 4), dq8(w[q], t));
}

// ================================================================ main kernel
constexpr int BMC = 128;  // activation rows per CTA and half (256 per pair)
constexpr int BNC = 128;  // weight columns decoded per CTA
constexpr int BT = 256;   // output columns of a pair tile (its rows: 256 * H)
constexpr int BK = 64;
constexpr int A_BYTES = BMC * BK * 2;  // 16 KB per 128-row activation tile
constexpr int W_BYTES = BNC * BK * 2;  // 16 KB
constexpr int STG_BYTES = 32 * 32 * 2;  // one warp's 32 rows x 32 columns of bf16 output
constexpr int SKB = 8;                  // 16 KB buffers of stream-K partials a finisher keeps in flight
constexpr int C_BYTES = BNC * BK / 2;  // 4 KB
// Warp roles: 0-3 epilogue (TMEM lane quarters), 5 TMEM owner and MMA issuer, 9 TMA producer,
// 4, 6, 7, 8, 10, 11, 12, 14 NF4 decoders, 13 idle.  A warp stalled issuing tcgen05.mma (or a TMA)
// holds back the shared-memory traffic of the other warps of its SM sub-partition (warp % 4):
// decoders beside the MMA issuer ran about four times slower than the rest (2700 against 650
// cycles per stage, measured on B200) and set the pace of every stage.  So the issuing warps share
// sub-partition 1 and the decoders take the other three.
constexpr int DQ_WARPS = 8;
constexpr int NTHREADS = 15 * 32;
constexpr int W_MMA = 5, W_TMA = 9;
__device__ __forceinline__ bool is_decoder(int warp) { return warp >= 4 && (warp & 3) != 1; }
// decoder index 0 .. 7 of a decoder warp (4 -> 0, 6 -> 1, 7 -> 2, 8 -> 3, 10 -> 4, 11 -> 5, 12 -> 6, 14 -> 7)
__device__ __forceinline__ int decoder_index(int warp) { return warp - 4 - (warp > 5) - (warp > 9) - (warp > 13); }

// H = 256-row halves per pair tile.  H = 1: six stages and two accumulator
// buffers, so the epilogue of one tile overlaps the main loop of the next.
// H = 2: a 512 x 256 tile whose two halves share every decoded weight tile
// (half the decode work per FLOP); both accumulators fill TMEM, four stages.
template <int H>
struct PCfg {
  static constexpr int NST = H == 1 ? 6 : 4;
  static constexpr int NBUF = H == 1 ? 2 : 1;
  static constexpr int A_STAGE = H * A_BYTES;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_W = OFF_A + NST * A_STAGE;
  static constexpr int OFF_C = OFF_W + NST * W_BYTES;
  static constexpr int OFF_BAR = OFF_C + NST * C_BYTES;
  // H = 2: the epilogue stages each warp's 32 x 32 output chunk (bf16, 64-byte swizzle) in one of
  // two 2 KB buffers per warp for a TMA store, the residual arriving there by TMA (one mbarrier
  // per buffer)
  static constexpr bool STG = H == 2;
  static constexpr int NBAR = 3 * NST + 2 * NBUF + 1 + SKB + (STG ? 8 : 0);
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
  static constexpr int OFF_STG = (OFF_MISC + 128 + 1023) / 1024 * 1024;
  static constexpr int SMEM_BYTES = (STG ? OFF_STG + 4 * 2 * STG_BYTES : OFF_MISC + 128) + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(NBUF * H * BT <= 512, "TMEM columns");
};

struct Seg {
  const float* absmax;
  __nv_bfloat16* y;          // FWD output [M, n]
  const __nv_bfloat16* res;  // FWD residual [M, n] or null (may alias y)
  int n;                     // rows of W
  int first;                 // FWD: first n-tile of the segment; DX: first contraction block
  int rope;                  // FWD: rotate this segment's output (heads of rope_hd columns)
};

struct Params {
  Seg seg[3];
  int nseg, M, K;
  int lora;          // 1: one LoRA contraction block follows the weight blocks
  int nkb;           // weight contraction blocks per tile
  int mtiles, tiles;
  __nv_bfloat16* dx;  // DX output [M, K]
  float cb[16];
  // FWD: rotate-half RoPE of the segments marked rope, position = row % rope_seq,
  // cos / sin from the table [rope_seq][rope_hd / 2] (rope_hd 64, 128 or 256)
  const float2* rope;
  int rope_seq, rope_hd;
  // stream-K: the first dp_tiles tiles (whole rounds) go to the clusters
  // whole, in the usual order; the weight blocks of the others are cut into
  // one contiguous range per cluster, and a range that ends inside a tile
  // leaves an fp32 partial that the cluster finishing the tile adds in cluster
  // order (see piece_at)
  int streamk, dp_tiles;
  float* part;                  // per (cluster, CTA): [H x 8 column chunks][8 float4][128 rows] float4
  unsigned long long* flags;    // per (cluster, CTA): the epoch once its partial is written
  unsigned long long epoch;     // unique per launch
};

struct Maps {
  CUtensorMap a[3];   // FWD: x [M, K]; DX: dy of each segment [M, n]  (box 64 x 128 rows, 128B swizzle)
  CUtensorMap c[3];   // packed codes of each segment: FWD box 32 B x 128 rows; DX box 64 B x 64 rows
  CUtensorMap la[3];  // LoRA block, activation side: FWD s*U of each segment [M, 64]; DX s*G [M, 64]
  CUtensorMap lb[3];  // LoRA block, weight side: FWD B of each segment, padded [n, 64]; DX A^T of all
                      // segments side by side [K, 64]
  CUtensorMap y[3];    // output (H = 2 epilogue stores): FWD y of each segment [M, n]; DX dx [M, K] in y[0]
                       // (box 32 x 32 rows, 64B swizzle)
  CUtensorMap res[3];  // FWD residual of each segment [M, n] (same box), where there is one
};

__device__ __forceinline__ int seg_of_block(const Params& p, int i) {
  int sg = 0;
  while (sg + 1 < p.nseg && i >= p.seg[sg + 1].first) ++sg;
  return sg;
}

// The j-th piece of work of cluster c of ncl: tile t, weight blocks [k0, k1)
// (plus the LoRA block when k1 == nkb).  Whole tiles: c, c + ncl, ...  With
// stream-K the whole tiles stop at dp_tiles; then comes the cluster's range
// [W c / ncl, W (c+1) / ncl) of the W = (tiles - dp_tiles) x nkb remaining
// blocks, walked from its last tile to its first, so that a range ending
// inside a tile writes that tile's partial first and the cluster that
// finishes the tile, whose range starts inside it, reaches it last.
__device__ __forceinline__ int64_t sk_bound(const Params& p, int c, int ncl) {
  return (int64_t)(p.tiles - p.dp_tiles) * p.nkb * c / ncl;
}
__device__ __forceinline__ bool piece_at(const Params& p, int c, int ncl, int j, int& t, int& k0, int& k1) {
  const int whole = p.streamk ? p.dp_tiles : p.tiles;
  if (c + j * ncl < whole) {
    t = c + j * ncl;
    k0 = 0;
    k1 = p.nkb;
    return true;
  }
  if (!p.streamk) return false;
  j -= (whole - c + ncl - 1) / ncl;  // the cluster's whole tiles come first
  const int64_t lo = sk_bound(p, c, ncl), hi = sk_bound(p, c + 1, ncl);
  if (hi <= lo) return false;
  const int tr = (int)((hi - 1) / p.nkb) - j;  // tile index within the stream-K part
  if ((int64_t)tr < lo / p.nkb) return false;
  const int64_t base = (int64_t)tr * p.nkb;
  t = p.dp_tiles + tr;
  k0 = (int)(max(lo, base) - base);
  k1 = (int)(min(hi, base + p.nkb) - base);
  return true;
}

template <int MODE, int H>
__device__ __forceinline__ void tile_at(const Params& p, int t, int& m0, int& sg, int& n0) {
  const int mt = t % p.mtiles, nt = t / p.mtiles;
  m0 = mt * BT * H;
  sg = 0;
  if (MODE == FWD) {
    while (sg + 1 < p.nseg && nt >= p.seg[sg + 1].first) ++sg;
    n0 = (nt - p.seg[sg].first) * BT;
  } else {
    n0 = nt * BT;
  }
}


// bf16 output of 32 columns (chunk c) of row m of a tile whose first column is n0, with the residual (FWD)
// A finisher that has seen the partials of clusters [c_lo, cid) for its rank clears their flags
// once every epilogue thread is past its wait (each flag has this one reader).  Every flag is 0
// again when the launch ends, so a launch replayed with the same epoch (a CUDA graph) cannot take
// a flag left from an earlier replay for its own.
__device__ __forceinline__ void clear_flags(const Params& p, int c_lo, int cid, unsigned rank) {
  for (int c2 = c_lo; c2 < cid; ++c2)
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p.flags + c2 * 2 + (int)rank), "l"(0ull) : "memory");
}

// The epilogue's hand-back of a TMEM accumulator: every epilogue thread of the CTA is past its
// last load of it; one thread clears the stream-K flags it consumed and arrives on the leader's
// tempty barrier.
__device__ __forceinline__ void release_acc(const Params& p, int cw, int cid, unsigned rank, int e,
                                            uint64_t* tempty_b) {
  tc_fence_before();
  named_bar_sync(1, 128);
  if (e == 0) {
    clear_flags(p, cw, cid, rank);
    mbar_arrive_cluster(cluster_addr(tempty_b, 0));
  }
}

// One lane's row of a staged 32 x 32 output chunk: the accumulator values v (plus the residual row
// at r_addr when res) rounded once to bf16 and written at s_addr (both rows of 64-byte-swizzled
// boxes, 16-byte piece q at (q ^ (row / 2 % 4)) * 16; r_addr may equal s_addr).
__device__ __forceinline__ void stage_chunk(float (&v)[32], bool res, uint32_t r_addr, uint32_t s_addr, int lane) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t sw = (uint32_t)(q ^ ((lane >> 1) & 3)) << 4;
    float* x = v + q * 8;
    if (res) {
      const uint4 rv = ld_shared_v4(r_addr + sw);
      x[0] += bf16lo(rv.x);
      x[1] += bf16hi(rv.x);
      x[2] += bf16lo(rv.y);
      x[3] += bf16hi(rv.y);
      x[4] += bf16lo(rv.z);
      x[5] += bf16hi(rv.z);
      x[6] += bf16lo(rv.w);
      x[7] += bf16hi(rv.w);
    }
    st_shared_v4(s_addr + sw, make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                         pack_bf16x2(x[6], x[7])));
  }
}

// The residual of row m's 32-column chunk c (FWD with a residual): four 16-byte words of bf16
// (the residual may alias y: each address is read before it is written).
template <int MODE>
__device__ __forceinline__ void load_res_chunk(const Params& p, int sg, int n0, int ncols, int m, int c,
                                               uint4 (&r)[4]) {
  if (MODE != FWD || m >= p.M) return;
  const Seg& S = p.seg[sg];
  if (!S.res) return;
#pragma unroll
  for (int gq = 0; gq < 4; ++gq) {
    const int col = n0 + c * 32 + gq * 8;
    if (col < ncols) r[gq] = *reinterpret_cast<const uint4*>(S.res + (int64_t)m * S.n + col);
  }
}

// One epilogue warp's 32 rows (from row0) of a finished 32-column chunk c through the warp's
// staging buffers (512-row tiles): the residual added per row from global memory (FWD), then
// staged in buffer nst & 1 and stored by TMA; nothing for rows past M.  All lanes call it.
template <int MODE>
__device__ __forceinline__ void staged_store(const Params& p, const CUtensorMap* ymap, int sg, int n0, int ncols,
                                             int row0, int c, float (&v)[32], uint8_t* stg, uint32_t& nst, int lane) {
  const int b = (int)(nst++ & 1u);
  if (lane == 0) bulk_wait_read<0>();  // every earlier store (a pair's included) has read its buffer
  __syncwarp();
  if (row0 >= p.M) return;  // warp-uniform
  if (MODE == FWD && p.seg[sg].res) {
    uint4 r[4] = {};
    load_res_chunk<MODE>(p, sg, n0, ncols, row0 + lane, c, r);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float* x = v + q * 8;
      x[0] += bf16lo(r[q].x);
      x[1] += bf16hi(r[q].x);
      x[2] += bf16lo(r[q].y);
      x[3] += bf16hi(r[q].y);
      x[4] += bf16lo(r[q].z);
      x[5] += bf16hi(r[q].z);
      x[6] += bf16lo(r[q].w);
      x[7] += bf16hi(r[q].w);
    }
  }
  const uint32_t s0 = smem_u32(stg + b * STG_BYTES) + (uint32_t)lane * 64;
  stage_chunk(v, false, s0, s0, lane);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(ymap, stg + b * STG_BYTES, n0 + c * 32, row0);
    bulk_commit();
  }
}

template <int MODE>
__device__ __forceinline__ void store_chunk(const Params& p, int sg, int n0, int ncols, int m, int c, float (&v)[32]) {
  if (m >= p.M) return;
#pragma unroll
  for (int gq = 0; gq < 4; ++gq) {
    const int col = n0 + c * 32 + gq * 8;
    if (col >= ncols) continue;
    float* x = v + gq * 8;
    if (MODE == FWD) {
      const Seg& S = p.seg[sg];
      const int64_t off = (int64_t)m * S.n + col;
      if (S.res) {
        const uint4 rv = *reinterpret_cast<const uint4*>(S.res + off);
        x[0] += bf16lo(rv.x);
        x[1] += bf16hi(rv.x);
        x[2] += bf16lo(rv.y);
        x[3] += bf16hi(rv.y);
        x[4] += bf16lo(rv.z);
        x[5] += bf16hi(rv.z);
        x[6] += bf16lo(rv.w);
        x[7] += bf16hi(rv.w);
      }
      *reinterpret_cast<uint4*>(S.y + off) = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                                                        pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
    } else {
      *reinterpret_cast<uint4*>(p.dx + (int64_t)m * p.K + col) =
          make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                     pack_bf16x2(x[6], x[7]));
    }
  }
}

template <int MODE, int H>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    nf4_pair_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Params p) {
  using C = PCfg<H>;
  constexpr int NST = C::NST, NBUF = C::NBUF;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + NST;
  uint64_t* cfull = empty + NST;
  uint64_t* tfull = cfull + NST;
  uint64_t* tempty = tfull + NBUF;
  uint64_t* drain = tempty + NBUF;
  uint64_t* sbar = drain + 1;   // [SKB]: stream-K partials pulled into the idle stages (finisher's last piece)
  uint64_t* rbar = sbar + SKB;  // [4 x 2] (H = 2): residual chunks landing in the epilogue's staging buffers
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);

  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cid = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1 + 2 * DQ_WARPS);  // leader's producer + every decoder warp of the pair
      mbar_init(&empty[s], 1);
      mbar_init(&cfull[s], 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2);  // one epilogue arrival per CTA
    }
    mbar_init(drain, 1);
    for (int b = 0; b < SKB; ++b) mbar_init(&sbar[b], 1);
    if constexpr (C::STG)
      for (int b = 0; b < 8; ++b) mbar_init(&rbar[b], 1);
    fence_barrier_init();
  }
  if (warp == W_MMA) {
    tmem_alloc_pair(s_tmem, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == W_TMA) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      int t, k0, k1;
      for (int j = 0; ok && piece_at(p, cid, ncl, j, t, k0, k1); ++j) {
        int m0, sg, n0;
        tile_at<MODE, H>(p, t, m0, sg, n0);
        const int mrow = m0 + (int)rank * BMC, wcol = n0 + (int)rank * BNC;
        const int kend = k1 + (k1 == p.nkb ? p.lora : 0);
        for (int i = k0; i < kend; ++i, ++g) {
          const int s = (int)(g % NST);
          const uint32_t ph = (g / NST) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, 421)) {
            ok = false;
            break;
          }
          const uint32_t fl = cluster_addr(&full[s], 0);
          uint8_t* a_dst = smem + C::OFF_A + s * C::A_STAGE;
          if (i < p.nkb) {
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * H * A_BYTES);
            mbar_arrive_expect_tx(&cfull[s], (uint32_t)C_BYTES);
            uint8_t* c_dst = smem + C::OFF_C + s * C_BYTES;
            const int bs = (MODE == DX) ? seg_of_block(p, i) : 0;
            const int x = (MODE == DX) ? (i - p.seg[bs].first) * BK : i * BK;
#pragma unroll
            for (int h = 0; h < H; ++h) tma_load_2d_pair(a_dst + h * A_BYTES, &maps.a[bs], fl, x, mrow + h * BT);
            if (MODE == DX) tma_load_2d(c_dst, &maps.c[bs], &cfull[s], wcol / 2, x);
            else tma_load_2d(c_dst, &maps.c[sg], &cfull[s], i * (BK / 2), wcol);
          } else {
            // no codes for the LoRA block, but cfull[s] still completes one phase per
            // block, so that every barrier's parity follows the block counter
            mbar_arrive(&cfull[s]);
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * (H * A_BYTES + W_BYTES));
#pragma unroll
            for (int h = 0; h < H; ++h) tma_load_2d_pair(a_dst + h * A_BYTES, &maps.la[sg], fl, 0, mrow + h * BT);
            tma_load_2d_pair(smem + C::OFF_W + s * W_BYTES, &maps.lb[sg], fl, 0, wcol);
          }
        }
      }
    }
  } else if (warp == W_MMA) {
    // ---------------------------------------------------------------- MMA issuer (leader CTA)
    if (rank == 0 && lane == 0) {
      const uint32_t id_k = idesc_bf16(2 * BMC, BT, 0, 0);   // both operands K-major
      const uint32_t id_mn = idesc_bf16(2 * BMC, BT, 0, 1);  // DX weight tile: MN-major
      uint32_t g = 0;
      bool ok = true;
      int t, k0, k1;
      for (int j = 0; ok && piece_at(p, cid, ncl, j, t, k0, k1); ++j) {
        const int buf = j % NBUF;
        const uint32_t tph = (uint32_t)(j / NBUF) & 1u;
        if (!mbar_wait(&tempty[buf], tph ^ 1u, 521)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * H * BT);
        const int kend = k1 + (k1 == p.nkb ? p.lora : 0);
        for (int i = k0; i < kend; ++i, ++g) {
          const int s = (int)(g % NST);
          const uint32_t ph = (g / NST) & 1u;
          if (!mbar_wait(&full[s], ph, 522)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + C::OFF_A + s * C::A_STAGE);
          const uint32_t w_base = smem_u32(smem + C::OFF_W + s * W_BYTES);
          const bool mn = (MODE == DX) && i < p.nkb;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bd =
                mn ? smem_desc(w_base + kk * 2048, 8192, 1024, 2) : smem_desc(w_base + kk * 32, 16, 1024, 2);
#pragma unroll
            for (int h = 0; h < H; ++h)
              tc_mma_pair(d + (uint32_t)(h * BT), smem_desc(a_base + h * A_BYTES + kk * 32, 16, 1024, 2), bd,
                          mn ? id_mn : id_k, (i != k0 || kk != 0));
          }
          tc_commit_pair_mc(&empty[s], 0x3);
        }
        if (ok) tc_commit_pair_mc(&tfull[buf], 0x3);
      }
      if (!ok) {
        tc_commit_pair(drain);
        mbar_wait(drain, 0, 523);
      }
    }
  } else if (is_decoder(warp)) {
    // ---------------------------------------------------------------- NF4 decoders
    const int t = decoder_index(warp) * 32 + lane;  // 0 .. 255
    const int KB = p.K / 64;
    uint32_t g = 0;
    bool ok = true;
    int tt, k0, k1;
    for (int j = 0; ok && piece_at(p, cid, ncl, j, tt, k0, k1); ++j) {
      int m0, sg, n0;
      tile_at<MODE, H>(p, tt, m0, sg, n0);
      const int wcol = n0 + (int)rank * BNC;
      const int kend = k1 + (k1 == p.nkb ? p.lora : 0);
      if (MODE == FWD) {
        // thread -> (row, half): consecutive lanes read consecutive 16-byte code
        // chunks and write conflict-free swizzled chunks
        const int row = t >> 1, half = t & 1;
        const Seg& S = p.seg[sg];
        const int n = wcol + row;
        const bool valid = n < S.n;
        const float* arow = S.absmax + (int64_t)(valid ? n : 0) * KB;
        // 16-byte absmax loads need every row start 16-byte aligned (the ABI promises 4)
        const bool vec = (KB % 4) == 0 && (reinterpret_cast<uintptr_t>(S.absmax) & 15) == 0;
        float4 acur = make_float4(0.f, 0.f, 0.f, 0.f), anext = acur;
        float s0 = 0.f, s1 = 0.f, s2 = 0.f;
        if (valid) {
          const int q0 = k0 & ~3;  // the float4 group of the piece's first block
          if (vec) {
            if (q0 < KB) acur = __ldg(reinterpret_cast<const float4*>(arow + q0));
            if (q0 + 4 < KB) anext = __ldg(reinterpret_cast<const float4*>(arow + q0 + 4));
          } else {
            if (k0 < KB) s0 = __ldg(arow + k0);
            if (k0 + 1 < KB) s1 = __ldg(arow + k0 + 1);
            if (k0 + 2 < KB) s2 = __ldg(arow + k0 + 2);
          }
        }
        for (int i = k0; i < kend; ++i, ++g) {
          const int s = (int)(g % NST);
          const uint32_t ph = (g / NST) & 1u;
          const uint32_t fl = cluster_addr(&full[s], 0);
          if (i < p.nkb) {
            const int q = i & 3;
            const float a = vec ? (q == 0 ? acur.x : q == 1 ? acur.y : q == 2 ? acur.z : acur.w) : s0;
            if (!__all_sync(0xffffffffu, mbar_wait(&cfull[s], ph, 631))) {
              ok = false;
              break;
            }
            const uint4 c = *reinterpret_cast<const uint4*>(smem + C::OFF_C + s * C_BYTES + t * 16);
            store_half_row(smem_u32(smem + C::OFF_W + s * W_BYTES) + row * 128, row, half, c, dq_table(valid ? a : 0.0f, p.cb));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(fl);
            if (valid) {
              if (vec) {
                if (q == 3) {
                  acur = anext;
                  if (i + 5 < KB) anext = __ldg(reinterpret_cast<const float4*>(arow + i + 5));
                }
              } else {
                s0 = s1;
                s1 = s2;
                if (i + 3 < KB) s2 = __ldg(arow + i + 3);
              }
            }
          } else {
            // LoRA block: its weight-side tile comes by TMA; arrive once the producer
            // has claimed the stage (cfull[s] completes without bytes for this block)
            if (!__all_sync(0xffffffffu, mbar_wait(&cfull[s], ph, 632))) {
              ok = false;
              break;
            }
            if (lane == 0) mbar_arrive_cluster(fl);
          }
        }
      } else {
        // DX stage tile: 64 contraction rows (n) x 128 output columns (k) = 64 x 2
        // blocks; thread -> (k chunk, row, half) so that the 8 lanes of each
        // store phase write 8 different swizzled chunks of 4 rows of one chunk
        const int kc = t >> 7, nl = (t & 127) >> 1, half = t & 1;
        const int kcol = wcol + kc * 64;
        auto absmax_of = [&](int i) {
          const int bs = seg_of_block(p, i);
          const Seg& S = p.seg[bs];
          const int nrow = (i - S.first) * BK + nl;
          return (nrow < S.n && kcol < p.K) ? __ldg(S.absmax + (int64_t)nrow * KB + kcol / 64) : 0.0f;
        };
        // absmax of the next four blocks in flight (global-load latency > one block)
        float a0 = k0 < p.nkb ? absmax_of(k0) : 0.0f;
        float a1 = k0 + 1 < p.nkb ? absmax_of(k0 + 1) : 0.0f;
        float a2 = k0 + 2 < p.nkb ? absmax_of(k0 + 2) : 0.0f;
        float a3 = k0 + 3 < p.nkb ? absmax_of(k0 + 3) : 0.0f;
        for (int i = k0; i < kend; ++i, ++g) {
          const int s = (int)(g % NST);
          const uint32_t ph = (g / NST) & 1u;
          const uint32_t fl = cluster_addr(&full[s], 0);
          if (i < p.nkb) {
            const float a = a0;
            a0 = a1;
            a1 = a2;
            a2 = a3;
            a3 = i + 4 < p.nkb ? absmax_of(i + 4) : 0.0f;
            if (!__all_sync(0xffffffffu, mbar_wait(&cfull[s], ph, 633))) {
              ok = false;
              break;
            }
            const uint4 c = *reinterpret_cast<const uint4*>(smem + C::OFF_C + s * C_BYTES + nl * (BNC / 2) + kc * 32 +
                                                            half * 16);
            store_half_row(smem_u32(smem + C::OFF_W + s * W_BYTES) + kc * 8192 + nl * 128, nl, half, c, dq_table(a, p.cb));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(fl);
          } else {
            if (!__all_sync(0xffffffffu, mbar_wait(&cfull[s], ph, 634))) {
              ok = false;
              break;
            }
            if (lane == 0) mbar_arrive_cluster(fl);
          }
        }
      }
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------------- epilogue (warps 0-3)
    const int e = threadIdx.x;  // TMEM lane = row within the CTA's 128
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    constexpr int PART_FLOATS = H * (BT / 32) * 128 * 32;  // one CTA's accumulator
    uint32_t rph = 0;          // H = 2 staging: parity of the warp's residual barrier
    uint32_t nst = 0;          // staged stores of the single-chunk paths (buffer nst & 1)
    bool stg_ok = true;        // false once a residual wait ran out: nothing more is stored
    int t, k0, k1;
    for (int j = 0; piece_at(p, cid, ncl, j, t, k0, k1); ++j) {
      int m0, sg, n0;
      tile_at<MODE, H>(p, t, m0, sg, n0);
      const int buf = j % NBUF;
      const uint32_t tph = (uint32_t)(j / NBUF) & 1u;
      if constexpr (C::STG) {
        // the tile's residual, needed only after its products, is brought into L2 meanwhile
        if (MODE == FWD && lane == 0 && k1 == p.nkb && p.seg[sg].res) {
          const int wrow = m0 + (int)rank * BMC + warp * 32;
          for (int h = 0; h < H; ++h)
            if (wrow + h * BT < p.M)
              for (int c = 0; c < BT / 32 && n0 + c * 32 < p.seg[sg].n; ++c)
                tma_prefetch_l2_2d(&maps.res[sg], n0 + c * 32, wrow + h * BT);
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], tph, 731))) break;
      tc_fence_after();
      if (k1 < p.nkb) {
        // the range ends inside this tile: park the fp32 partial, then publish it
        // row e's 32 values of chunk hc as 8 float4, each at [hc][q][e]: a warp's store covers 512
        // contiguous bytes
        float4* dst = reinterpret_cast<float4*>(p.part + (int64_t)(cid * 2 + (int)rank) * PART_FLOATS);
        for (int hc = 0; hc < H * (BT / 32); ++hc) {
          float v[32];
          tmem_ld32(tmem + lane_base + (uint32_t)(buf * H * BT + hc * 32), v);
          tc_wait_ld();
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[((int64_t)hc * 8 + q) * 128 + e] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
        __threadfence();
        tc_fence_before();
        named_bar_sync(1, 128);
        if (e == 0) {
          asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p.flags + cid * 2 + (int)rank), "l"(p.epoch)
                       : "memory");
          mbar_arrive_cluster(cluster_addr(&tempty[buf], 0));
        }
        continue;
      }
      // clusters whose ranges end inside this tile, before this one's: their partials, in cluster order
      int cfirst = cid;
      bool seen = true;  // every awaited flag held this launch's epoch
      if (p.streamk && k0 > 0) {
        const int64_t tstart = (int64_t)(t - p.dp_tiles) * p.nkb;
        while (cfirst > 0 && sk_bound(p, cfirst, ncl) > tstart) --cfirst;
        // ranges are not empty when stream-K runs (at least 4 blocks per cluster, see launch_pair); an
        // empty one would leave no partial, so it is skipped here and below all the same
        while (cfirst < cid && sk_bound(p, cfirst + 1, ncl) == sk_bound(p, cfirst, ncl)) ++cfirst;
        for (int c2 = cfirst; c2 < cid; ++c2) {
          if (sk_bound(p, c2 + 1, ncl) == sk_bound(p, c2, ncl)) continue;  // an empty range leaves no partial
          const unsigned long long* f = p.flags + c2 * 2 + (int)rank;
          unsigned long long v = 0;
          const uint64_t t0 = globaltimer();
          while (true) {
            asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(f) : "memory");
            if (v == p.epoch) break;
            if (globaltimer() - t0 > LSQ_WAIT_NS) {
              report(LSQ_ETIMEOUT, 735);
              seen = false;
              break;
            }
          }
        }
      }
      const int cw = seen ? cfirst : cid;  // flags [cw, cid) are cleared at the end of this tile
      // 16 columns (piece 0 or 1) of two chunks hca, hcb of this tile's accumulator plus the
      // partials of the clusters before this one, added in the same order as the 32-column path
      // below; the two chunks' loads are issued together
      auto acc16x2 = [&](int hca, int hcb, int piece, float (&va)[16], float (&vb)[16]) {
        tmem_ld16(tmem + lane_base + (uint32_t)((buf * H + hca / (BT / 32)) * BT + (hca % (BT / 32)) * 32 + piece * 16),
                  va);
        tmem_ld16(tmem + lane_base + (uint32_t)((buf * H + hcb / (BT / 32)) * BT + (hcb % (BT / 32)) * 32 + piece * 16),
                  vb);
        if (cfirst == cid) {
          tc_wait_ld();
          return;
        }
        bool first = true;
        for (int c2 = cfirst; c2 < cid; ++c2) {
          if (c2 > cfirst && sk_bound(p, c2 + 1, ncl) == sk_bound(p, c2, ncl)) continue;
          const float4* base = reinterpret_cast<const float4*>(p.part + (int64_t)(c2 * 2 + (int)rank) * PART_FLOATS);
          const float4* sa = base + ((int64_t)hca * 8 + piece * 4) * 128 + e;
          const float4* sb = base + ((int64_t)hcb * 8 + piece * 4) * 128 + e;
          float4 a[4], b[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            a[q] = __ldcg(sa + q * 128);
            b[q] = __ldcg(sb + q * 128);
          }
          if (first) tc_wait_ld();
          first = false;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            va[4 * q] += a[q].x;
            va[4 * q + 1] += a[q].y;
            va[4 * q + 2] += a[q].z;
            va[4 * q + 3] += a[q].w;
            vb[4 * q] += b[q].x;
            vb[4 * q + 1] += b[q].y;
            vb[4 * q + 2] += b[q].z;
            vb[4 * q + 3] += b[q].w;
          }
        }
      };
      const int ncols = (MODE == FWD) ? p.seg[sg].n : p.K;
      // A finisher that adds partials on its last piece (stream-K, 512-row tiles) pulls them into
      // its idle activation stages with bulk copies: per 32-column chunk up to 4 partials of 16 KB
      // per round, two rounds in flight, instead of one round trip per partial per chunk.  The
      // partials are added in the same order as below, so the two paths agree bit for bit.
      bool bulk = false;
      if constexpr (H == 2) {
        int tn, k0n, k1n;
        bulk = cfirst < cid && cid - cfirst <= 16 && !piece_at(p, cid, ncl, j + 1, tn, k0n, k1n);
        for (int c2 = cfirst; bulk && c2 < cid; ++c2) bulk = sk_bound(p, c2 + 1, ncl) > sk_bound(p, c2, ncl);
      }
      const bool rope_seg = MODE == FWD && p.seg[sg].rope;
      if (bulk) {
        // units u = (chunk k, contributor i), chunk-major: the 16 KB of contributor i's partial for
        // chunk k, bulk-copied into one of SKB buffers of the idle activation stages, SKB units in
        // flight (so the L2 round trips overlap); added in cluster order, as in the path below
        const int P = cid - cfirst;
        const int cvalid = min(BT / 32, (ncols - n0 + 31) / 32);
        const int nunits = H * cvalid * P;
        uint8_t* stage = smem + C::OFF_A;  // SKB x 16 KB of the activation stages, idle now
        const float* part0 = p.part + (int64_t)(cfirst * 2 + (int)rank) * PART_FLOATS;
        auto issue = [&](int uu) {  // thread e == 0
          const int k = uu / P, i = uu % P;
          const int hc = (k / cvalid) * (BT / 32) + k % cvalid;
          mbar_arrive_expect_tx(&sbar[uu % SKB], 16384u);
          bulk_g2s(stage + (uu % SKB) * 16384, part0 + (int64_t)i * 2 * PART_FLOATS + (int64_t)hc * 4096, 16384u,
                   &sbar[uu % SKB]);
        };
        if (e == 0) {
          fence_proxy_async_all();  // the partials were published to this thread's acquires above
          for (int uu = 0; uu < min(SKB, nunits); ++uu) issue(uu);
        }
        bool okb = true;  // false once a wait ran out: every thread still passes every barrier, nothing is stored
        int u = 0;
        for (int k = 0; k < H * cvalid; ++k) {
          const int h = k / cvalid, c = k % cvalid;
          float v[32];
          tmem_ld32(tmem + lane_base + (uint32_t)((buf * H + h) * BT + c * 32), v);
          for (int i = 0; i < P; ++i, ++u) {
            okb = okb && mbar_wait(&sbar[u % SKB], (uint32_t)(u / SKB) & 1u, 736);
            if (i == 0) tc_wait_ld();
            if (okb) {
              const float4* sb = reinterpret_cast<const float4*>(stage + (u % SKB) * 16384) + e;
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 a = sb[q * 128];
                v[4 * q] += a.x;
                v[4 * q + 1] += a.y;
                v[4 * q + 2] += a.z;
                v[4 * q + 3] += a.w;
              }
            }
            // buffer u % SKB is read (unit u + SKB may refill it); a wait that ran out anywhere stops all
            okb = named_bar_and(1, 128, okb);
            if (e == 0 && okb && u + SKB < nunits) issue(u + SKB);
          }
          if (!__all_sync(0xffffffffu, okb)) continue;
          if (rope_seg) {  // the sum goes back into the accumulator for the RoPE epilogue below
            tmem_st32(tmem + lane_base + (uint32_t)((buf * H + h) * BT + c * 32), v);
          } else if constexpr (C::STG) {
            staged_store<MODE>(p, &maps.y[MODE == FWD ? sg : 0], sg, n0, ncols, m0 + h * BT + (int)rank * BMC + warp * 32,
                               c, v, smem + C::OFF_STG + warp * 2 * STG_BYTES, nst, lane);
          } else {
            store_chunk<MODE>(p, sg, n0, ncols, m0 + h * BT + (int)rank * BMC + e, c, v);
          }
        }
        if (rope_seg) {
          tc_wait_st();
          cfirst = cid;  // the accumulator holds the tile's whole sum now
        } else {
          tc_fence_before();
          named_bar_sync(1, 128);
          if (e == 0) {
            clear_flags(p, cw, cid, rank);
            mbar_arrive_cluster(cluster_addr(&tempty[buf], 0));
          }
          continue;
        }
      }
      if constexpr (C::STG) {
        if (rope_seg && cfirst == cid) {
          // RoPE with the staged stores of the path below: the two 32-column chunks of a head
          // whose columns pair up (c and c + hd/64) are loaded together, rotated in fp32 (the
          // same arithmetic as the unstaged RoPE path below) and rounded once, staged and stored
          // by TMA.
          const int hc32 = p.rope_hd / 32, heads = BT / p.rope_hd;
          const float* inv = reinterpret_cast<const float*>(p.rope) + (int64_t)p.rope_seq * p.rope_hd;
          const int wrow = m0 + (int)rank * BMC + warp * 32;
          uint8_t* stg = smem + C::OFF_STG + warp * 2 * STG_BYTES;
          const int npairs = H * heads * (hc32 / 2);
          int pi = 0;
          for (int h = 0; h < H; ++h) {
            const int row = wrow + h * BT;
            const float pos = (float)((row + lane) % p.rope_seq);
            for (int hh = 0; hh < heads; ++hh) {
              for (int cl = 0; cl < hc32 / 2; ++cl, ++pi) {
                const int ca = hh * hc32 + cl, cb = ca + hc32 / 2;
                float va[32], vb[32];
                tmem_ld32(tmem + lane_base + (uint32_t)((buf * H + h) * BT + ca * 32), va);
                tmem_ld32(tmem + lane_base + (uint32_t)((buf * H + h) * BT + cb * 32), vb);
                if (lane == 0) bulk_wait_read<0>();  // the last pair's stores have read both buffers
                __syncwarp();
                tc_wait_ld_regs(va);
                tc_wait_ld_regs(vb);
                if (pi + 1 == npairs) release_acc(p, cw, cid, rank, e, &tempty[buf]);
                if (row >= p.M || n0 + ca * 32 >= ncols) continue;  // warp-uniform
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  const float2 t = rope_cs(pos * __ldg(inv + cl * 32 + i));
                  const float a = va[i], b = vb[i];
                  va[i] = a * t.x - b * t.y;
                  vb[i] = b * t.x + a * t.y;
                }
                const uint32_t s0 = smem_u32(stg) + (uint32_t)lane * 64;
                stage_chunk(va, false, s0, s0, lane);
                stage_chunk(vb, false, s0 + STG_BYTES, s0 + STG_BYTES, lane);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                  tma_store_2d(&maps.y[sg], stg, n0 + ca * 32, row);
                  tma_store_2d(&maps.y[sg], stg + STG_BYTES, n0 + cb * 32, row);
                  bulk_commit();
                }
              }
            }
          }
          continue;
        }
      }
      if (rope_seg) {
        // RoPE in the epilogue: column i of a head pairs with column i + hd/2, which sits hd/64
        // chunks of 32 further on in the same accumulator; both are rotated in fp32 (the
        // accumulator plus earlier clusters' partials) and rounded once.  The angle of each
        // pair is its row's position times the frequency, its cosine and sine computed here
        // (rope_cs) from the table's per-frequency tail: no per-position table traffic.
        const int hc32 = p.rope_hd / 32, half = p.rope_hd / 2, heads = BT / p.rope_hd;
        const float* inv = reinterpret_cast<const float*>(p.rope) + (int64_t)p.rope_seq * p.rope_hd;
        for (int fb = 0; fb < half / 16; ++fb) {
          const int cl = fb / 2, piece = fb % 2;
          for (int h = 0; h < H; ++h) {
            const int m = m0 + h * BT + (int)rank * BMC + e;
            const float pos = (float)(m % p.rope_seq);
            for (int hh = 0; hh < heads; ++hh) {
              const int c = hh * hc32 + cl;
              if (n0 + c * 32 >= ncols) continue;
              float x1[16], x2[16];
              acc16x2(h * (BT / 32) + c, h * (BT / 32) + c + hc32 / 2, piece, x1, x2);
              if (m >= p.M) continue;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 t = rope_cs(pos * __ldg(inv + fb * 16 + i));
                const float a = x1[i], b = x2[i];
                x1[i] = a * t.x - b * t.y;
                x2[i] = b * t.x + a * t.y;
              }
              const Seg& S = p.seg[sg];
              __nv_bfloat16* y1 = S.y + (int64_t)m * S.n + n0 + c * 32 + piece * 16;
              __nv_bfloat16* y2 = y1 + half;
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                *reinterpret_cast<uint4*>(y1 + 8 * u) =
                    make_uint4(pack_bf16x2(x1[8 * u], x1[8 * u + 1]), pack_bf16x2(x1[8 * u + 2], x1[8 * u + 3]),
                               pack_bf16x2(x1[8 * u + 4], x1[8 * u + 5]), pack_bf16x2(x1[8 * u + 6], x1[8 * u + 7]));
                *reinterpret_cast<uint4*>(y2 + 8 * u) =
                    make_uint4(pack_bf16x2(x2[8 * u], x2[8 * u + 1]), pack_bf16x2(x2[8 * u + 2], x2[8 * u + 3]),
                               pack_bf16x2(x2[8 * u + 4], x2[8 * u + 5]), pack_bf16x2(x2[8 * u + 6], x2[8 * u + 7]));
              }
            }
          }
        }
        tc_fence_before();
        named_bar_sync(1, 128);
        if (e == 0) {
          clear_flags(p, cw, cid, rank);
          mbar_arrive_cluster(cluster_addr(&tempty[buf], 0));
        }
        continue;
      }
      if constexpr (C::STG) {
        if (cfirst == cid) {
          // The whole sum is in TMEM.  Each warp takes its 32 rows two 32-column chunks at a time:
          // both TMEM loads in flight together, then each chunk written to one of the warp's two
          // staging buffers (bf16, 64-byte swizzle: 16-byte piece q of row i at
          // i * 64 + (q ^ (i / 2 % 4)) * 16, conflict-free with one row per lane) and stored by
          // one lane with TMA, so the output leaves as whole lines.  The accumulator goes back to
          // the MMA issuer as soon as its last chunks are in registers.  A residual comes in by
          // TMA: when no piece follows this one, the tile's whole residual at once into the idle
          // activation stages (box (h, c) of warp w at ((w * H + h) * 8 + c) * 2 KB), else each
          // pair's boxes into the staging buffers just ahead of their use.
          const int si = MODE == FWD ? sg : 0;
          const bool res = MODE == FWD && p.seg[si].res != nullptr;
          const int cvalid = min(BT / 32, (ncols - n0 + 31) / 32);  // chunks of each half inside n
          const int wrow = m0 + (int)rank * BMC + warp * 32;        // the warp's first row in half 0
          uint8_t* stg = smem + C::OFF_STG + warp * 2 * STG_BYTES;
          uint64_t* rb = &rbar[warp * 2];
          int tn, k0n, k1n;
          const bool res_all = res && !piece_at(p, cid, ncl, j + 1, tn, k0n, k1n);
          uint8_t* rall = smem + C::OFF_A + warp * H * (BT / 32) * STG_BYTES;
          bool rpend = false;  // a residual load on rb not yet waited for
          if (res_all && stg_ok) {
            if (lane == 0) {
              uint32_t bytes = 0;
              for (int h = 0; h < H; ++h)
                if (wrow + h * BT < p.M) bytes += (uint32_t)cvalid * STG_BYTES;
              if (bytes) {
                mbar_arrive_expect_tx(rb, bytes);
                for (int h = 0; h < H; ++h)
                  if (wrow + h * BT < p.M)
                    for (int c = 0; c < cvalid; ++c)
                      tma_load_2d(rall + (h * (BT / 32) + c) * STG_BYTES, &maps.res[si], rb, n0 + c * 32, wrow + h * BT);
              }
            }
            rpend = wrow < p.M;  // warp-uniform: half 0's rows decide whether anything was loaded
          }
          for (int h = 0; h < H; ++h) {
            const int row = wrow + h * BT;
            for (int c = 0; c < cvalid; c += 2) {
              const bool two = c + 1 < cvalid;
              float va[32], vb[32];
              // (chunk c + 1 < BT / 32 always exists in TMEM; past n it is loaded but not stored)
              tmem_ld32(tmem + lane_base + (uint32_t)((buf * H + h) * BT + c * 32), va);
              tmem_ld32(tmem + lane_base + (uint32_t)((buf * H + h) * BT + (c + 1) * 32), vb);
              const bool pair_res = res && !res_all && stg_ok && row < p.M;
              if (lane == 0) {
                bulk_wait_read<0>();  // the last pair's stores have read both buffers
                if (pair_res) {
                  mbar_arrive_expect_tx(rb, (two ? 2u : 1u) * STG_BYTES);
                  tma_load_2d(stg, &maps.res[si], rb, n0 + c * 32, row);
                  if (two) tma_load_2d(stg + STG_BYTES, &maps.res[si], rb, n0 + (c + 1) * 32, row);
                }
              }
              __syncwarp();
              tc_wait_ld_regs(va);
              tc_wait_ld_regs(vb);
              if (h + 1 == H && c + 2 >= cvalid) release_acc(p, cw, cid, rank, e, &tempty[buf]);
              if (row >= p.M) continue;  // the warp's rows are all past M (warp-uniform)
              if ((pair_res || rpend) && stg_ok) {
                stg_ok = __all_sync(0xffffffffu, mbar_wait(rb, rph & 1u, 737));
                rph ^= 1u;
                rpend = false;
              }
              if (!stg_ok) continue;
              const uint32_t lrow = (uint32_t)lane * 64;
              const uint32_t s0 = smem_u32(stg) + lrow;
              const uint32_t r0 = res_all ? smem_u32(rall + (h * (BT / 32) + c) * STG_BYTES) + lrow : s0;
              stage_chunk(va, res, r0, s0, lane);
              if (two) stage_chunk(vb, res, r0 + STG_BYTES, s0 + STG_BYTES, lane);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&maps.y[si], stg, n0 + c * 32, row);
                if (two) tma_store_2d(&maps.y[si], stg + STG_BYTES, n0 + (c + 1) * 32, row);
                bulk_commit();
              }
            }
          }
          continue;
        }
      }
      for (int hc = 0; hc < H * (BT / 32); ++hc) {
        const int h = hc / (BT / 32), c = hc % (BT / 32);
        if (n0 + c * 32 >= ncols) continue;
        const int m = m0 + h * BT + (int)rank * BMC + e;
        float v[32];
        tmem_ld32(tmem + lane_base + (uint32_t)((buf * H + h) * BT + c * 32), v);
        if (cfirst == cid) {
          tc_wait_ld();
        } else {
          // the first contributor's partial is loaded while the TMEM load completes
          const float4* src0 = reinterpret_cast<const float4*>(p.part + (int64_t)(cfirst * 2 + (int)rank) * PART_FLOATS) +
                               (int64_t)hc * 8 * 128 + e;
          float4 a[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) a[q] = __ldcg(src0 + q * 128);
          tc_wait_ld();
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            v[4 * q] += a[q].x;
            v[4 * q + 1] += a[q].y;
            v[4 * q + 2] += a[q].z;
            v[4 * q + 3] += a[q].w;
          }
          for (int c2 = cfirst + 1; c2 < cid; ++c2) {
            if (sk_bound(p, c2 + 1, ncl) == sk_bound(p, c2, ncl)) continue;
            const float4* src = reinterpret_cast<const float4*>(p.part + (int64_t)(c2 * 2 + (int)rank) * PART_FLOATS) +
                                (int64_t)hc * 8 * 128 + e;
#pragma unroll
            for (int q = 0; q < 8; ++q) a[q] = __ldcg(src + q * 128);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              v[4 * q] += a[q].x;
              v[4 * q + 1] += a[q].y;
              v[4 * q + 2] += a[q].z;
              v[4 * q + 3] += a[q].w;
            }
          }
        }
        if constexpr (C::STG)
          staged_store<MODE>(p, &maps.y[MODE == FWD ? sg : 0], sg, n0, ncols, m0 + h * BT + (int)rank * BMC + warp * 32, c,
                             v, smem + C::OFF_STG + warp * 2 * STG_BYTES, nst, lane);
        else
          store_chunk<MODE>(p, sg, n0, ncols, m, c, v);
      }
      tc_fence_before();
      named_bar_sync(1, 128);
      if (e == 0) {
        clear_flags(p, cw, cid, rank);
        mbar_arrive_cluster(cluster_addr(&tempty[buf], 0));
      }
    }
    if constexpr (C::STG) {
      if (lane == 0) bulk_wait_all();  // the staged stores are written before the CTA exits
    }
  }

  tc_fence_before();
  cluster_sync_all();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ================================================================ rank-r products: U = X A^T, G = dY B
// Split-K tcgen05 GEMM with a narrow N, reduced inside a thread-block cluster:
// the S CTAs of a cluster (S <= 8) take one 128-row tile of one problem and
// split its contraction; each parks its fp32 partial [128 x np] in its own
// shared memory, then rank k adds the S partials of rows [k*128/S, ...) in
// rank order through distributed shared memory (a fixed order: results do not
// depend on timing) and writes the outputs:
//   FWD (one problem, segment q in columns q*rp ..): u_out[q] [M, r] fp32 (if
//        given) and s*U of segment q as bf16 [M, 64], zero in columns >= r;
//        meanwhile the epilogue warps of every CTA, idle until their MMAs
//        finish, write the padded copies of B that the main GEMM reads.
//   DX  (problem q = segment q): s*G as bf16 [M, 64] with segment q in columns
//        q*rp .. q*rp + rp - 1 and zeros from nseg*rp on.
namespace ldn {
constexpr int BM = 128, BK = 64, NST = 4, NMAX = 192;
constexpr int A_BYTES = BM * BK * 2;    // 16 KB
constexpr int B_BYTES = NMAX * BK * 2;  // 24 KB
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + NST * A_BYTES;
constexpr int NBAR = 2 * NST + 1;
// the weight-side stages hold np_max rows of 128 bytes: sized per launch (bst bytes each), so that
// narrow problems leave room for two or three CTAs per SM
__host__ __device__ constexpr int off_bar(int bst) { return OFF_B + NST * bst; }
__host__ __device__ constexpr int smem_bytes(int bst) { return off_bar(bst) + 8 * NBAR + 16 + 1024; }
constexpr int OFF_BAR = off_bar(B_BYTES);
constexpr int SMEM_BYTES = smem_bytes(B_BYTES);
constexpr int NTHREADS = 192;
constexpr int TARGET_CTAS = 296;
constexpr int MAX_SPLITS = 8;  // portable cluster size
static_assert(BM * (NMAX + 4) * 4 <= OFF_BAR, "partial tile must fit the stage buffers");

struct Prob {
  int nkb;   // contraction blocks of 64 (the last may be partial: zero-filled)
  int kbps;  // blocks per split: split k covers [k*kbps, min(nkb, (k+1)*kbps))
  int nsub;  // weight-side maps wl[first .. first + nsub), rp rows each
  int first;
};
struct Params {
  Prob pr[3];
  int nprob, M, r, rp, dx, nseg;
  int bst;  // bytes of one weight-side stage (np of the widest problem x 128), a multiple of 1024
  float s;
  float* out32[3];          // FWD: U of each segment (or null)
  __nv_bfloat16* out16[3];  // FWD: s*U of each segment [M, 64]; DX: s*G [M, 64] in out16[0]
  const __nv_bfloat16* B[3];  // FWD: LoRA B of each segment [n, r] ...
  __nv_bfloat16* Bpad[3];     // ... and its padded copy [n, 64]
  int64_t nB[3];
};
struct Maps {
  CUtensorMap in[3];  // activation side of each problem [M, Kr] (box 64 x 128 rows, 128B swizzle)
  CUtensorMap wl[3];  // weight side [rows, Kr] (box 64 x rp rows; rows past the tensor read as zero)
};

// plain load from a cluster peer's shared memory (after a cluster barrier: the
// compiler may batch these, so a thread's loads from all peers overlap)
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t caddr) {
  float4 v;
  asm("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(caddr));
  return v;
}

__global__ void __launch_bounds__(NTHREADS, 1) lora_down_kernel(const __grid_constant__ Maps maps,
                                                                const __grid_constant__ Params p) {
  const int pi = blockIdx.z;
  const Prob& P = p.pr[pi];
  const int split = blockIdx.y;  // rank in the cluster (the cluster spans y)
  const int S = gridDim.y;
  const int kb0 = split * P.kbps;
  const int nk = max(0, min(P.nkb, kb0 + P.kbps) - kb0);
  const int np = P.nsub * p.rp;
  const int ldp = np + 4;  // row stride of the parked partial (floats): 16-byte rows, no bank conflicts
  const int m0 = blockIdx.x * BM;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + off_bar(p.bst));
  uint64_t* empty = full + NST;
  uint64_t* done = empty + NST;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + off_bar(p.bst) + 8 * NBAR);
  float* park = reinterpret_cast<float*>(smem);  // [128][ldp], over the stage buffers once the MMAs are done
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ncols = np <= 32 ? 32u : np <= 64 ? 64u : np <= 128 ? 128u : 256u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < nk; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, 441)) break;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(A_BYTES + np * 128));
        const int x = (kb0 + i) * BK;
        tma_load_2d(smem + OFF_A + s * A_BYTES, &maps.in[pi], &full[s], x, m0);
        for (int q = 0; q < P.nsub; ++q)
          tma_load_2d(smem + OFF_B + s * p.bst + q * p.rp * 128, &maps.wl[P.first + q], &full[s], x, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16(BM, np, 0, 0);
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        if (!mbar_wait(&full[s], ph, 541)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + OFF_A + s * A_BYTES);
        const uint32_t b_base = smem_u32(smem + OFF_B + s * p.bst);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          tc_mma(tmem, smem_desc(a_base + kk * 32, 16, 1024, 2), smem_desc(b_base + kk * 32, 16, 1024, 2), id,
                 (i | kk) != 0);
        tc_commit(&empty[s]);
      }
      tc_commit(done);  // also the drain when the loop stopped early; completes at once if nk == 0
      if (!ok) mbar_wait(done, 0, 542);
    }
  } else {
    // epilogue warps 2-5: TMEM lane quarter = warp % 4
    const int qd = warp & 3;
    const int e = qd * 32 + lane;  // row of the tile
    if (!p.dx) {
      // padded copies of B, spread over every CTA of the grid while its MMAs run
      const int64_t cta = ((int64_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
      const int64_t stride = (int64_t)gridDim.x * gridDim.y * gridDim.z * 128;
      for (int q = 0; q < p.nseg; ++q) {
        const int64_t total = p.nB[q] * 8;  // 16-byte chunks of Bpad[q]
        for (int64_t c = cta * 128 + (threadIdx.x - 64); c < total; c += stride) {
          const int64_t n = c >> 3;
          const int j0 = (int)(c & 7) * 8;
          float v[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) v[t] = j0 + t < p.r ? __bfloat162float(p.B[q][n * p.r + j0 + t]) : 0.0f;
          *reinterpret_cast<uint4*>(p.Bpad[q] + n * 64 + j0) =
              make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                         pack_bf16x2(v[6], v[7]));
        }
      }
    }
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(done, 0, 741));
    if (ok && nk > 0) tc_fence_after();
    for (int c = 0; c < np / 16; ++c) {
      float v[16];
      if (ok && nk > 0) {
        tmem_ld16(tmem + lane_base + (uint32_t)(c * 16), v);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int t = 0; t < 16; ++t) v[t] = 0.0f;
      }
      float4* dst = reinterpret_cast<float4*>(park + e * ldp + c * 16);
#pragma unroll
      for (int t = 0; t < 4; ++t) dst[t] = make_float4(v[4 * t], v[4 * t + 1], v[4 * t + 2], v[4 * t + 3]);
    }
  }
  tc_fence_before();
  cluster_sync_all();  // every CTA's partial is parked
  if (warp >= 2) {
    // rank k adds the cluster's partials for its own slice of rows, in rank order
    const int per = (BM + S - 1) / S, r0 = split * per, r1 = min(BM, r0 + per);
    const int nch = np / 8;  // 8-column chunks per row
    const int t = threadIdx.x - 64;
    for (int it = t; it < (r1 - r0) * nch; it += 128) {
      const int e = r0 + it / nch, c = (it % nch) * 8;
      const int64_t m = m0 + e;
      if (m >= p.M) continue;
      const uint32_t local = smem_u32(park + e * ldp + c);
      float4 x0[MAX_SPLITS], x1[MAX_SPLITS];
#pragma unroll
      for (int k = 0; k < MAX_SPLITS; ++k) {
        if (k < S) {
          uint32_t a;
          asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(local), "r"(k));
          x0[k] = ld_dsmem_f4(a);
          x1[k] = ld_dsmem_f4(a + 16);
        }
      }
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < MAX_SPLITS; ++k) {
        if (k < S) {
          v[0] += x0[k].x; v[1] += x0[k].y; v[2] += x0[k].z; v[3] += x0[k].w;
          v[4] += x1[k].x; v[5] += x1[k].y; v[6] += x1[k].z; v[7] += x1[k].w;
        }
      }
      const int q = c / p.rp, j0 = c % p.rp;  // segment and rank of the first column
      const uint4 o = make_uint4(pack_bf16x2(p.s * v[0], p.s * v[1]), pack_bf16x2(p.s * v[2], p.s * v[3]),
                                 pack_bf16x2(p.s * v[4], p.s * v[5]), pack_bf16x2(p.s * v[6], p.s * v[7]));
      if (p.dx) {
        *reinterpret_cast<uint4*>(p.out16[0] + m * 64 + pi * p.rp + j0) = o;
      } else {
        *reinterpret_cast<uint4*>(p.out16[q] + m * 64 + j0) = o;
        if (p.out32[q])
          for (int u = 0; u < 8; ++u)
            if (j0 + u < p.r) p.out32[q][m * p.r + j0 + u] = v[u];
      }
    }
    // zero padding of the bf16 operands for the same rows
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int e = r0 + t; e < r1; e += 128) {
      const int64_t m = m0 + e;
      if (m >= p.M) continue;
      if (p.dx) {
        if (pi == 0)
          for (int c = p.nseg * p.rp; c < 64; c += 8) *reinterpret_cast<uint4*>(p.out16[0] + m * 64 + c) = z;
      } else {
        for (int q = 0; q < p.nseg; ++q)
          for (int c = p.rp; c < 64; c += 8) *reinterpret_cast<uint4*>(p.out16[q] + m * 64 + c) = z;
      }
    }
  }
  cluster_sync_all();  // every CTA keeps its shared memory until the others have read it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// splits (cluster size) so that about TARGET_CTAS CTAs run; at most 8 and at most the blocks
static int plan_splits(int ctas_per_split, int nkb_max) {
  int s = (TARGET_CTAS + ctas_per_split - 1) / ctas_per_split;
  return std::max(1, std::min(s, std::min(MAX_SPLITS, nkb_max)));
}
static size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// Padded copies of the LoRA operands for the backward (the forward's padded B
// is written inside lora_down_kernel):
//   job q < nseg: Bt_q [rp, n_q] = B_q^T, zero rows >= r
//   job nseg: At [K, 64] = A_q^T of every segment q in columns q*rp .., zero elsewhere
//   job nseg + 1 + q: SU_q [M, 64] = bf16(s * U_q) in columns < r, zero elsewhere
struct Pad {
  const __nv_bfloat16* A[3];
  const __nv_bfloat16* B[3];
  const float* U[3];
  __nv_bfloat16* Bt[3];
  __nv_bfloat16* SU[3];
  __nv_bfloat16* At;
  int64_t n[3];
  int64_t K, M;
  int nseg, r, rp;
  float s;
};

__global__ void __launch_bounds__(256) lora_pad(const __grid_constant__ Pad P) {
  const int job = blockIdx.y;
  const bool at = job == P.nseg;
  const bool su = job > P.nseg;
  const int64_t total = su ? P.M * 64 : at ? P.K * 64 : (int64_t)P.rp * P.n[job];
  const __nv_bfloat16 zero = __float2bfloat16_rn(0.0f);
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    if (su) {
      const int q = job - P.nseg - 1;
      const int64_t m = idx / 64;
      const int c = (int)(idx % 64);
      P.SU[q][idx] = c < P.r ? __float2bfloat16_rn(P.s * P.U[q][m * P.r + c]) : zero;
    } else if (at) {
      const int64_t k = idx / 64;
      const int c = (int)(idx % 64), q = c / P.rp, j = c % P.rp;
      P.At[idx] = (q < P.nseg && j < P.r) ? P.A[q][(int64_t)j * P.K + k] : zero;
    } else {
      const int64_t j = idx / P.n[job], n = idx % P.n[job];
      P.Bt[job][idx] = j < P.r ? P.B[job][n * P.r + j] : zero;
    }
  }
}

}  // namespace ldn

// ---------------------------------------------------------------- launch helpers
template <int MODE, int H>
static lsq_status launch_pair_h(const Maps& maps, const Params& p, int ncl, cudaStream_t stream) {
  nf4_pair_kernel<MODE, H><<<2 * ncl, NTHREADS, PCfg<H>::SMEM_BYTES, stream>>>(maps, p);
  LSQ_LAUNCH_CHECK("nf4_pair_kernel");
  return LSQ_OK;
}

// Pair clusters that fit on the GPU at once (74 on 148 SMs), queried once per device.
static lsq_status max_pair_clusters(int* out) {
  static int max_clusters[64] = {0};
  int dev = 0;
  LSQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(LSQ_EUNSUPPORTED, "nf4 GEMM: device %d out of range", dev);
  if (!max_clusters[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(nf4_pair_kernel<FWD, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      PCfg<1>::SMEM_BYTES));
    LSQ_CUDA_TRY(cudaFuncSetAttribute(nf4_pair_kernel<DX, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      PCfg<1>::SMEM_BYTES));
    LSQ_CUDA_TRY(cudaFuncSetAttribute(nf4_pair_kernel<FWD, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      PCfg<2>::SMEM_BYTES));
    LSQ_CUDA_TRY(cudaFuncSetAttribute(nf4_pair_kernel<DX, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      PCfg<2>::SMEM_BYTES));
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(2 * num_sms());
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = PCfg<1>::SMEM_BYTES;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, nf4_pair_kernel<FWD, 1>, &cfg) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      n = num_sms() / 2;
    }
    max_clusters[dev] = n;
  }
  *out = max_clusters[dev];
  return LSQ_OK;
}

// Workspace for stream-K: 4 KB of per-(cluster, CTA) flags, then one 512 x 256
// fp32 partial per cluster (256 KB per CTA).
static size_t sk_region_bytes() {
  int n = 0;
  if (max_pair_clusters(&n) != LSQ_OK || n < 1) {
    (void)cudaGetLastError();
    n = 74;
  }
  return 4096 + (size_t)n * 2 * (size_t)(2 * (BT / 32) * 128 * 32 * sizeof(float));
}
// unique per launch within the process (a partial's flag holds its launch's value; its reader
// clears it, see clear_flags, so a replayed launch may reuse the value)
static unsigned long long next_epoch() {
  static std::atomic<unsigned long long> counter{
      (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() * 0x9E3779B97F4A7C15ull};
  return ++counter;
}

// Rows per pair tile: 512 (H = 2) halves the NF4 decode work per FLOP but
// leaves no second accumulator for the epilogue to overlap; 256 (H = 1) keeps
// the overlap.  With a stream-K workspace (sk_ws, at least sk_region_bytes())
// the last one or two rounds' worth of tiles can be shared out as equal
// ranges of weight blocks instead (stream-K, H = 2; see piece_at).  The fix-up
// of the tiles split between clusters (a 256 KB partial written and read back
// per CTA, one more accumulator hand-over) costs about 0.4 of a tile-time on
// B200, so it is used where it saves more: at 2048 rows, 96 tiles of 512 rows
// on 74 clusters take 1.3 + 0.4 tile-times instead of 2 rounds (q/k/v forward:
// 138 -> 126 us), 448 take 6.05 + 0.4 instead of 7 (gate/up: 423 -> 390 us),
// 224 take 3.03 + 0.4 instead of 4 (down's dX: 292 -> 257 us with the adapter
// kernels), while 64 tiles (one round, 10 clusters idle) stay whole.
// Otherwise pick the tile height with fewer rounds of whole tiles, an H = 2
// tile costing 1.25 times an H = 1 tile (measured on B200 at the 8B shapes:
// 1.4-1.7x the TFLOP/s of H = 1 at 2048 rows).  LSQ_NF4_TILE_ROWS=256|512
// forces whole tiles of that height.
template <int MODE>
static lsq_status launch_pair(const Maps& maps, Params p, int ntiles_n, char* sk_ws, size_t sk_bytes,
                              cudaStream_t stream) {
  int ncl_max = 0;
  lsq_status st = max_pair_clusters(&ncl_max);
  if (st != LSQ_OK) return st;
  const char* force = getenv("LSQ_NF4_TILE_ROWS");
  const int64_t tiles2 = (int64_t)((p.M + 2 * BT - 1) / (2 * BT)) * ntiles_n;
  p.streamk = 0;
  const double rounds_sk = (double)tiles2 / ncl_max + 0.4;
  const double rounds_whole = (double)((tiles2 + ncl_max - 1) / ncl_max);
  const int64_t dp = std::max<int64_t>(0, tiles2 / ncl_max - 1) * ncl_max;
  // LSQ_NF4_STREAMK=0 never shares tiles out, =1 does wherever it can (a tuning override)
  const char* skenv = getenv("LSQ_NF4_STREAMK");
  const int skmode = skenv ? atoi(skenv) : -1;
  const bool sk_can = !force && sk_ws && sk_bytes >= sk_region_bytes() && p.M >= 2 * BT && p.nkb >= 8 &&
                      (tiles2 - dp) * p.nkb >= 4 * (int64_t)ncl_max;
  const bool sk_pays = 2 * tiles2 >= ncl_max && rounds_sk < 0.97 * rounds_whole;
  static const bool plan_log = getenv("LSQ_NF4_PLAN_LOG") != nullptr;   // prints each call's tile plan
  // Few tiles (under half a round of 512-row tiles, e.g. 512 tokens): let S clusters share each
  // tile (ncl = tiles x S, so each finisher adds at most about S partials).  Cost model in us,
  // from B200 microbenchmarks at the 3B shapes: about 8 of fixed cost per launch, 1.0 per
  // 64-wide weight block of a 512-row tile (0.73 for a 256-row one), and about 5 per partial the
  // finisher adds (bulk copies into its idle stages; 10 with one round trip per partial).
  // Only long contractions (at least 128 weight blocks, where it was measured to pay: 1.5-2.3x at
  // the 3B shapes' 172 and 344 blocks) take it.
  if (!force && skmode != 0 && sk_ws && sk_bytes >= sk_region_bytes() && p.M >= 2 * BT && p.nkb >= 128 &&
      2 * tiles2 < ncl_max) {
    const int64_t tiles1 = (int64_t)((p.M + BT - 1) / BT) * ntiles_n;
    const double whole1 = 8.0 + (double)((tiles1 + ncl_max - 1) / ncl_max) * p.nkb * 0.73;
    const double whole2 = 8.0 + (double)((tiles2 + ncl_max - 1) / ncl_max) * p.nkb * 1.0;
    const double whole = std::min(whole1, whole2);
    int sbest = 1;
    double cbest = whole;
    const char* splitenv = getenv("LSQ_NF4_SK_SPLIT");   // forces S (a tuning override)
    for (int S = 2; S * tiles2 <= ncl_max; ++S) {
      if (tiles2 * p.nkb < 4 * (int64_t)S * tiles2) break;  // at least 4 blocks per cluster
      const double c = 8.0 + (double)p.nkb / S + 5.0 * (S - 1);
      if (splitenv ? S == atoi(splitenv) : c < 0.85 * cbest) {
        cbest = c;
        sbest = S;
      }
    }
    if (sbest > 1) {
      const int ncl_s = (int)(tiles2 * sbest);
      if (plan_log)
        fprintf(stderr, "nf4 plan: mode %d M %d tiles %lld (512 rows) nkb %d: stream-K over %d clusters (%d per "
                "tile)\n", MODE, p.M, (long long)tiles2, p.nkb, ncl_s, sbest);
      p.streamk = 1;
      p.dp_tiles = 0;
      p.flags = reinterpret_cast<unsigned long long*>(sk_ws);
      p.part = reinterpret_cast<float*>(sk_ws + 4096);
      p.epoch = next_epoch();
      p.mtiles = (p.M + 2 * BT - 1) / (2 * BT);
      p.tiles = p.mtiles * ntiles_n;
      return launch_pair_h<MODE, 2>(maps, p, ncl_s, stream);
    }
  }
  if (sk_can && skmode != 0 && (skmode == 1 || sk_pays)) {
    if (plan_log)
      fprintf(stderr, "nf4 plan: mode %d M %d tiles %lld (512 rows) nkb %d: stream-K, %lld whole tiles\n", MODE, p.M,
              (long long)tiles2, p.nkb, (long long)dp);
    p.streamk = 1;
    p.dp_tiles = (int)dp;  // whole tiles for all but the last one or two rounds' worth
    p.flags = reinterpret_cast<unsigned long long*>(sk_ws);
    p.part = reinterpret_cast<float*>(sk_ws + 4096);
    p.epoch = next_epoch();
    p.mtiles = (p.M + 2 * BT - 1) / (2 * BT);
    p.tiles = p.mtiles * ntiles_n;
    return launch_pair_h<MODE, 2>(maps, p, ncl_max, stream);
  }
  int64_t best = -1;
  int hbest = 1;
  for (int h = 1; h <= 2; ++h) {
    const int64_t tiles = (int64_t)((p.M + BT * h - 1) / (BT * h)) * ntiles_n;
    const int64_t rounds = (tiles + ncl_max - 1) / ncl_max;
    const int64_t cost = rounds * (h == 1 ? 4 : 5);
    if (best < 0 || cost < best) {
      best = cost;
      hbest = h;
    }
  }
  if (const char* e = force) {
    const int rows = atoi(e);
    if (rows == 256) hbest = 1;
    if (rows == 512) hbest = 2;
  }
  p.mtiles = (p.M + BT * hbest - 1) / (BT * hbest);
  p.tiles = p.mtiles * ntiles_n;
  const int ncl = std::min(p.tiles, ncl_max);
  if (plan_log)
    fprintf(stderr, "nf4 plan: mode %d M %d tiles %d (%d rows) nkb %d: whole tiles on %d clusters%s\n", MODE, p.M,
            p.tiles, 256 * hbest, p.nkb, ncl, sk_can ? "" : " (no stream-K: not possible)");
  return hbest == 2 ? launch_pair_h<MODE, 2>(maps, p, ncl, stream) : launch_pair_h<MODE, 1>(maps, p, ncl, stream);
}

// one cluster of `splits` CTAs per (row tile, problem)
static lsq_status launch_down(const ldn::Maps& maps, const ldn::Params& p_in, int splits, cudaStream_t stream) {
  static int configured[64] = {0};
  int dev = 0;
  LSQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(ldn::lora_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      ldn::SMEM_BYTES));
    LSQ_CUDA_TRY(cudaFuncSetAttribute(ldn::lora_down_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                      cudaSharedmemCarveoutMaxShared));
    configured[dev] = 1;
  }
  ldn::Params p = p_in;
  int np_max = 0;
  for (int i = 0; i < p.nprob; ++i) np_max = std::max(np_max, p.pr[i].nsub * p.rp);
  p.bst = np_max * 128;
  if (np_max < 16 || np_max > ldn::NMAX || p.bst % 1024 != 0) return fail(LSQ_EINVAL, "lora_down: rank width");
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)((p.M + ldn::BM - 1) / ldn::BM), (unsigned)splits, (unsigned)p.nprob);
  cfg.blockDim = dim3(ldn::NTHREADS);
  cfg.dynamicSmemBytes = ldn::smem_bytes(p.bst);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)splits;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  LSQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, ldn::lora_down_kernel, maps, p));
  return LSQ_OK;
}

// jobs 0 .. nseg-1: B^T of each segment; nseg: A^T of all segments; nseg+1 ..: s*U of each segment
static lsq_status launch_pad(const ldn::Pad& P, int64_t most, cudaStream_t stream, int jobs = -1) {
  int64_t g = (most + 255) / 256;
  if (g > 512) g = 512;
  if (g < 1) g = 1;
  ldn::lora_pad<<<dim3((unsigned)g, jobs > 0 ? jobs : 2 * P.nseg + 1), 256, 0, stream>>>(P);
  LSQ_LAUNCH_CHECK("lora_pad");
  return LSQ_OK;
}

static void fill_cb(Params& p) {
  const float* cb = codebook();
  for (int i = 0; i < 16; ++i) p.cb[i] = cb[i];
}

static lsq_status tmap_act(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, uint32_t box_outer) {
  return encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, (uint64_t)inner, (uint64_t)outer,
                        (uint64_t)inner * 2, 64, box_outer, CU_TENSOR_MAP_SWIZZLE_128B);
}
// an output (or residual) [rows, cols] bf16 as the H = 2 epilogue moves it: 32 x 32 boxes, 64B swizzle
static lsq_status tmap_out(CUtensorMap* m, const void* base, int64_t cols, int64_t rows) {
  return encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, (uint64_t)cols, (uint64_t)rows,
                        (uint64_t)cols * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

}  // namespace nf4g

// ================================================================ host paths
namespace tc {
using namespace lsq::nf4g;

static int rpad(int r) { return r > 0 ? (r + 15) / 16 * 16 : 0; }

static lsq_status nf4_checks(int64_t M, int64_t K, int32_t r, const char* who) {
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  if (M < 1 || M > (1 << 30)) return fail(LSQ_EINVAL, "%s: M out of range (%lld)", who, (long long)M);
  if (K < 64 || K % 64 != 0 || K > (1 << 30))
    return fail(LSQ_EINVAL, "%s: k_in must be a positive multiple of 64 (got %lld)", who, (long long)K);
  if (r < 0 || r > 64) return fail(LSQ_EINVAL, "%s: LoRA rank must be in [0, 64] (got %d)", who, r);
  return LSQ_OK;
}

static lsq_status check_weight(const lsq_nf4_weight& w, int64_t K, const char* who) {
  if (!w.codes || !w.absmax) return fail(LSQ_EINVAL, "%s: NULL weight pointer", who);
  if (w.k_in != K) return fail(LSQ_EINVAL, "%s: k_in mismatch (%lld vs %lld)", who, (long long)w.k_in, (long long)K);
  if (w.n_out < 8 || w.n_out % 8 != 0 || w.n_out > (1 << 30))
    return fail(LSQ_EINVAL, "%s: n_out must be a positive multiple of 8 (got %lld)", who, (long long)w.n_out);
  if (!aligned(w.codes, 16) || !aligned(w.absmax, 4))
    return fail(LSQ_EINVAL, "%s: codes must be 16-byte and absmax 4-byte aligned", who);
  return LSQ_OK;
}

// ---- forward: workspace = s*U per segment [M, 64] bf16 | padded B per segment [n, 64] bf16
struct FwdPlan {
  int splits, kbps;
  size_t su, bpad[3], total;
};
static FwdPlan fwd_plan(int nseg, int64_t M, int64_t K, const int64_t* n_out, int r) {
  (void)r;
  FwdPlan f;
  memset(&f, 0, sizeof(f));
  const int nkb = (int)(K / 64);
  const int mtiles = (int)((M + ldn::BM - 1) / ldn::BM);
  f.splits = ldn::plan_splits(mtiles, nkb);
  f.kbps = (nkb + f.splits - 1) / f.splits;
  f.su = ldn::round256((size_t)M * 64 * 2);
  f.total = (size_t)nseg * f.su;
  for (int i = 0; i < nseg; ++i) {
    f.bpad[i] = ldn::round256((size_t)n_out[i] * 64 * 2);
    f.total += f.bpad[i];
  }
  return f;
}

// ---- backward rank-r part: s*G bf16 [M, 64] | A^T side by side [K, 64] | B_q^T [rp, n_q] | s*U_q [M, 64]
struct BwdPlan {
  int splits;
  size_t sg, at, bt[3], su, total;
};
static BwdPlan bwd_plan(int nseg, int64_t M, int64_t K, const int64_t* n_out, int r) {
  BwdPlan b;
  memset(&b, 0, sizeof(b));
  const int rp = rpad(r);
  int nkb_max = 1;
  for (int i = 0; i < nseg; ++i) nkb_max = std::max(nkb_max, (int)((n_out[i] + 63) / 64));
  const int mtiles = (int)((M + ldn::BM - 1) / ldn::BM);
  b.splits = ldn::plan_splits(mtiles * nseg, nkb_max);
  b.sg = ldn::round256((size_t)M * 64 * 2);
  b.at = ldn::round256((size_t)K * 64 * 2);
  b.su = b.sg;
  b.total = b.sg + b.at + (size_t)nseg * b.su;
  for (int i = 0; i < nseg; ++i) {
    b.bt[i] = ldn::round256((size_t)rp * (size_t)n_out[i] * 2);
    b.total += b.bt[i];
  }
  return b;
}

// ---- rank state of one fused linear (the LoRA operands both passes read):
// s*U per segment [M, 64] | padded B per segment [n, 64] | B^T per segment [rp, n] | A^T side by side [K, 64]
struct StatePlan {
  size_t su, bpad[3], bt[3], at, total;
};
static StatePlan state_plan(int nseg, int64_t M, int64_t K, const int64_t* n_out, int r) {
  StatePlan sp;
  memset(&sp, 0, sizeof(sp));
  const int rp = rpad(r);
  sp.su = ldn::round256((size_t)M * 64 * 2);
  sp.at = ldn::round256((size_t)K * 64 * 2);
  sp.total = (size_t)nseg * sp.su + sp.at;
  for (int i = 0; i < nseg; ++i) {
    sp.bpad[i] = ldn::round256((size_t)n_out[i] * 64 * 2);
    sp.bt[i] = ldn::round256((size_t)rp * (size_t)n_out[i] * 2);
    sp.total += sp.bpad[i] + sp.bt[i];
  }
  return sp;
}
struct StatePtrs {
  __nv_bfloat16* su[3];
  __nv_bfloat16* bpad[3];
  __nv_bfloat16* bt[3];
  __nv_bfloat16* at;
};
static StatePtrs state_ptrs(void* state, int nseg, const StatePlan& sp) {
  StatePtrs q;
  memset(&q, 0, sizeof(q));
  char* cur = static_cast<char*>(state);
  for (int i = 0; i < nseg; ++i, cur += sp.su) q.su[i] = reinterpret_cast<__nv_bfloat16*>(cur);
  for (int i = 0; i < nseg; ++i) {
    q.bpad[i] = reinterpret_cast<__nv_bfloat16*>(cur);
    cur += sp.bpad[i];
  }
  for (int i = 0; i < nseg; ++i) {
    q.bt[i] = reinterpret_cast<__nv_bfloat16*>(cur);
    cur += sp.bt[i];
  }
  q.at = reinterpret_cast<__nv_bfloat16*>(cur);
  return q;
}

size_t bwd_rank_bytes(int nseg, int64_t M, int64_t K, const int64_t* n_out, int r) {
  return bwd_plan(nseg, M, K, n_out, r).total;
}

// s*G = s dY B of every segment side by side in bf16 [M, 64] (the dX GEMM's
// LoRA block and dA's operand), s*U of each segment in bf16 [M, 64] (dB's
// operand), and A^T of every segment side by side [K, 64]; ws starts with the
// layout of bwd_plan.  The bf16 pointers come back through sg / su / at.
lsq_status bwd_rank_part(int nseg, const lsq_nf4_weight* W, const void* const* dy, int64_t M, const void* const* A,
                         const void* const* B, const float* const* U, int r, float s, char* ws, __nv_bfloat16** sg,
                         __nv_bfloat16** su, __nv_bfloat16** at, cudaStream_t stream, const StatePtrs* state) {
  const int64_t K = W[0].k_in;
  const int rp = rpad(r);
  int64_t n_out[3];
  for (int i = 0; i < nseg; ++i) n_out[i] = W[i].n_out;
  const BwdPlan b = bwd_plan(nseg, M, K, n_out, r);
  char* cur = ws;
  *sg = reinterpret_cast<__nv_bfloat16*>(cur);
  cur += b.sg;
  *at = reinterpret_cast<__nv_bfloat16*>(cur);
  cur += b.at;
  __nv_bfloat16* bt[3];
  for (int i = 0; i < nseg; ++i) {
    bt[i] = reinterpret_cast<__nv_bfloat16*>(cur);
    cur += b.bt[i];
  }
  for (int i = 0; i < nseg; ++i) {
    su[i] = reinterpret_cast<__nv_bfloat16*>(cur);
    cur += b.su;
  }
  lsq_status st;
  if (state) {  // the forward left B^T, A^T and s*U: only G remains to compute
    *at = state->at;
    for (int i = 0; i < nseg; ++i) {
      bt[i] = state->bt[i];
      su[i] = state->su[i];
    }
  }
  ldn::Pad P;
  memset(&P, 0, sizeof(P));
  int64_t most = K * 64;
  for (int i = 0; i < nseg; ++i) {
    P.A[i] = static_cast<const __nv_bfloat16*>(A[i]);
    P.B[i] = static_cast<const __nv_bfloat16*>(B[i]);
    P.U[i] = U ? U[i] : nullptr;
    P.Bt[i] = bt[i];
    P.SU[i] = su[i];
    P.n[i] = n_out[i];
    most = std::max<int64_t>(most, (int64_t)rp * n_out[i]);
  }
  most = std::max<int64_t>(most, M * 64);
  P.At = *at;
  P.K = K;
  P.M = M;
  P.s = s;
  P.nseg = nseg;
  P.r = r;
  P.rp = rp;
  if (!state && (st = launch_pad(P, most, stream)) != LSQ_OK) return st;

  ldn::Maps maps;
  memset(&maps, 0, sizeof(maps));
  ldn::Params p;
  memset(&p, 0, sizeof(p));
  p.nprob = nseg;
  p.M = (int)M;
  p.r = r;
  p.rp = rp;
  p.dx = 1;
  p.nseg = nseg;
  p.s = s;
  p.out16[0] = *sg;
  for (int i = 0; i < nseg; ++i) {
    if ((st = tmap_act(&maps.in[i], dy[i], n_out[i], M, ldn::BM)) != LSQ_OK) return st;
    if ((st = tmap_act(&maps.wl[i], bt[i], n_out[i], rp, (uint32_t)rp)) != LSQ_OK) return st;
    ldn::Prob& pr = p.pr[i];
    pr.nkb = (int)((n_out[i] + 63) / 64);
    pr.kbps = (pr.nkb + b.splits - 1) / b.splits;
    pr.nsub = 1;
    pr.first = i;
  }
  return launch_down(maps, p, b.splits, stream);
}

// dX = sum_q dY_q deq(W_q) (+ (s G) A when sg != null)
lsq_status launch_dx(int nseg, const lsq_nf4_weight* W, const void* const* dy, int64_t M, const __nv_bfloat16* sg,
                     const __nv_bfloat16* at, void* dx, char* sk_ws, size_t sk_bytes, cudaStream_t stream) {
  const int64_t K = W[0].k_in;
  Params p;
  memset(&p, 0, sizeof(p));
  p.nseg = nseg;
  p.M = (int)M;
  p.K = (int)K;
  p.lora = sg ? 1 : 0;
  p.dx = static_cast<__nv_bfloat16*>(dx);
  fill_cb(p);
  Maps maps;
  memset(&maps, 0, sizeof(maps));
  int blocks = 0;
  lsq_status st;
  for (int i = 0; i < nseg; ++i) {
    Seg& g = p.seg[i];
    g.absmax = W[i].absmax;
    g.n = (int)W[i].n_out;
    g.first = blocks;
    blocks += (int)((W[i].n_out + BK - 1) / BK);
    if ((st = tmap_act(&maps.a[i], dy[i], W[i].n_out, M, BMC)) != LSQ_OK) return st;
    if ((st = encode_tmap_2d(&maps.c[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, W[i].codes, K / 2, W[i].n_out, K / 2,
                             BNC / 2, BK, CU_TENSOR_MAP_SWIZZLE_NONE)) != LSQ_OK)
      return st;
  }
  if (sg) {
    if ((st = tmap_act(&maps.la[0], sg, 64, M, BMC)) != LSQ_OK) return st;
    if ((st = tmap_act(&maps.lb[0], at, 64, K, BNC)) != LSQ_OK) return st;
  }
  if ((st = tmap_out(&maps.y[0], dx, K, M)) != LSQ_OK) return st;
  p.nkb = blocks;
  return launch_pair<DX>(maps, p, (int)((K + BT - 1) / BT), sk_ws, sk_bytes, stream);
}

}  // namespace tc
}  // namespace lsq

extern "C" size_t lsq_nf4_lora_fwd_workspace_size(int32_t nseg, int64_t M, int64_t k_in, const int64_t* n_out,
                                                  int32_t r) {
  if (nseg < 1 || nseg > 3 || r < 0 || r > 64 || M < 1 || k_in < 64 || !n_out) return 256;
  return (r > 0 ? lsq::tc::fwd_plan(nseg, M, k_in, n_out, r).total : 0) + lsq::nf4g::sk_region_bytes();
}

namespace lsq {
namespace tc {
using namespace lsq::nf4g;

// Argument checks shared by the forward entry points.
static lsq_status fwd_checks(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M,
                             const void* const* A, const void* const* B, int32_t r, const void* const* residual,
                             void* const* y, int64_t* ns, const char* who) {
  if (nseg < 1 || nseg > 3) return fail(LSQ_EINVAL, "%s: 1..3 segments (got %d)", who, nseg);
  if (!W || !x || !y) return fail(LSQ_EINVAL, "%s: NULL argument", who);
  const int64_t K = W[0].k_in;
  lsq_status st = nf4_checks(M, K, r, who);
  if (st != LSQ_OK) return st;
  if (!aligned(x, 16)) return fail(LSQ_EINVAL, "%s: x must be 16-byte aligned", who);
  for (int i = 0; i < nseg; ++i) {
    if ((st = check_weight(W[i], K, who)) != LSQ_OK) return st;
    ns[i] = W[i].n_out;
    if (!y[i] || !aligned(y[i], 16)) return fail(LSQ_EINVAL, "%s: y[%d] NULL or not 16-byte aligned", who, i);
    const void* res = residual ? residual[i] : nullptr;
    if (res && !aligned(res, 16)) return fail(LSQ_EINVAL, "%s: residual must be 16-byte aligned", who);
    if (r > 0) {
      if (!A || !B || !A[i] || !B[i]) return fail(LSQ_EINVAL, "%s: LoRA A/B NULL with r > 0", who);
      if (!aligned(A[i], 16) || !aligned(B[i], 2)) return fail(LSQ_EINVAL, "%s: LoRA A must be 16-byte aligned", who);
    }
  }
  return LSQ_OK;
}

// The forward proper.  su / bpad: where s*U and the padded B live (and are
// written when rank_part); bt / at: when non-null, B^T and A^T are written
// there too (the backward's operands); sk_ws: room for stream-K.
static lsq_status fwd_impl(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M, const void* const* A,
                           const void* const* B, int32_t r, float s, const void* const* residual, void* const* y,
                           float* const* u_out, __nv_bfloat16* const* su, __nv_bfloat16* const* bpad,
                           bool rank_part, __nv_bfloat16* const* bt, __nv_bfloat16* at, char* sk_ws,
                           size_t sk_bytes, cudaStream_t cs, const lsq_rope_spec* rope = nullptr) {
  const int64_t K = W[0].k_in;
  const int rp = rpad(r);
  int64_t ns[3];
  for (int i = 0; i < nseg; ++i) ns[i] = W[i].n_out;
  lsq_status st;
  Params p;
  memset(&p, 0, sizeof(p));
  p.nseg = nseg;
  p.M = (int)M;
  p.K = (int)K;
  p.lora = r > 0 ? 1 : 0;
  p.nkb = (int)(K / BK);
  fill_cb(p);
  if (rope) {
    p.rope = reinterpret_cast<const float2*>(rope->table);
    p.rope_seq = rope->seq;
    p.rope_hd = rope->hd;
  }
  Maps maps;
  memset(&maps, 0, sizeof(maps));
  if ((st = tmap_act(&maps.a[0], x, K, M, BMC)) != LSQ_OK) return st;
  int tiles_n = 0;
  for (int i = 0; i < nseg; ++i) {
    Seg& g = p.seg[i];
    g.absmax = W[i].absmax;
    g.y = static_cast<__nv_bfloat16*>(y[i]);
    g.res = static_cast<const __nv_bfloat16*>(residual ? residual[i] : nullptr);
    g.n = (int)W[i].n_out;
    g.first = tiles_n;
    g.rope = (rope && (rope->segments >> i) & 1) ? 1 : 0;
    tiles_n += (int)((W[i].n_out + BT - 1) / BT);
    if ((st = encode_tmap_2d(&maps.c[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, W[i].codes, K / 2, W[i].n_out, K / 2,
                             BK / 2, BNC, CU_TENSOR_MAP_SWIZZLE_NONE)) != LSQ_OK)
      return st;
    if ((st = tmap_out(&maps.y[i], g.y, g.n, M)) != LSQ_OK) return st;
    if (g.res && (st = tmap_out(&maps.res[i], g.res, g.n, M)) != LSQ_OK) return st;
  }
  if (r > 0) {
    if (rank_part) {
      const FwdPlan f = fwd_plan(nseg, M, K, ns, r);
      ldn::Maps dm;
      memset(&dm, 0, sizeof(dm));
      ldn::Params dp;
      memset(&dp, 0, sizeof(dp));
      if ((st = tmap_act(&dm.in[0], x, K, M, ldn::BM)) != LSQ_OK) return st;
      for (int i = 0; i < nseg; ++i) {
        if ((st = tmap_act(&dm.wl[i], A[i], K, r, (uint32_t)rp)) != LSQ_OK) return st;
        dp.out32[i] = u_out ? u_out[i] : nullptr;
        dp.out16[i] = su[i];
        dp.B[i] = static_cast<const __nv_bfloat16*>(B[i]);
        dp.Bpad[i] = bpad[i];
        dp.nB[i] = ns[i];
      }
      dp.nprob = 1;
      dp.M = (int)M;
      dp.r = r;
      dp.rp = rp;
      dp.dx = 0;
      dp.nseg = nseg;
      dp.s = s;
      dp.pr[0].nkb = (int)(K / 64);
      dp.pr[0].kbps = f.kbps;
      dp.pr[0].nsub = nseg;
      dp.pr[0].first = 0;
      if ((st = launch_down(dm, dp, f.splits, cs)) != LSQ_OK) return st;
      if (bt && at) {  // B^T and A^T for the backward: the transposition jobs of lora_pad
        ldn::Pad P;
        memset(&P, 0, sizeof(P));
        int64_t most = K * 64;
        for (int i = 0; i < nseg; ++i) {
          P.A[i] = static_cast<const __nv_bfloat16*>(A[i]);
          P.B[i] = static_cast<const __nv_bfloat16*>(B[i]);
          P.Bt[i] = bt[i];
          P.n[i] = ns[i];
          most = std::max<int64_t>(most, (int64_t)rp * ns[i]);
        }
        P.At = at;
        P.K = K;
        P.M = M;
        P.s = s;
        P.nseg = nseg;
        P.r = r;
        P.rp = rp;
        if ((st = launch_pad(P, most, cs, nseg + 1)) != LSQ_OK) return st;
      }
    }
    for (int i = 0; i < nseg; ++i) {
      if ((st = tmap_act(&maps.la[i], su[i], 64, M, BMC)) != LSQ_OK) return st;
      if ((st = tmap_act(&maps.lb[i], bpad[i], 64, ns[i], BNC)) != LSQ_OK) return st;
    }
  }
  return launch_pair<FWD>(maps, p, tiles_n, sk_ws, sk_bytes, cs);
}

}  // namespace tc
}  // namespace lsq

namespace lsq {
namespace tc {
// the workspace form of the fused forward (the rank-r operands rebuilt in the workspace), with optional RoPE
static lsq_status fwd_multi_ws(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M, const void* const* A,
                               const void* const* B, int32_t r, float s, const void* const* residual, void* const* y,
                               float* const* u_out, void* workspace, size_t workspace_bytes, lsq_cuda_stream stream,
                               const lsq_rope_spec* rope, const char* who);
}  // namespace tc
}  // namespace lsq

extern "C" lsq_status lsq_nf4_lora_fwd_multi(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M,
                                             const void* const* A, const void* const* B, int32_t r, float s,
                                             const void* const* residual, void* const* y, float* const* u_out,
                                             void* workspace, size_t workspace_bytes, lsq_cuda_stream stream) {
  return lsq::tc::fwd_multi_ws(nseg, W, x, M, A, B, r, s, residual, y, u_out, workspace, workspace_bytes, stream,
                               nullptr, "lsq_nf4_lora_fwd");
}

static lsq_status lsq::tc::fwd_multi_ws(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M,
                                        const void* const* A, const void* const* B, int32_t r, float s,
                                        const void* const* residual, void* const* y, float* const* u_out,
                                        void* workspace, size_t workspace_bytes, lsq_cuda_stream stream,
                                        const lsq_rope_spec* rope, const char* who) {
  using namespace lsq;
  int64_t ns[3];
  lsq_status st = tc::fwd_checks(nseg, W, x, M, A, B, r, residual, y, ns, who);
  if (st != LSQ_OK) return st;
  const int64_t K = W[0].k_in;
  const tc::FwdPlan f = tc::fwd_plan(nseg, M, K, ns, r);
  const size_t base = r > 0 ? f.total : 0;
  if (r > 0 && (!workspace || workspace_bytes < base || !aligned(workspace, 256)))
    return fail(LSQ_EINVAL, "%s: workspace needs %zu bytes, 256-byte aligned (got %zu)", who, base,
                workspace_bytes);
  // workspace: s*U per segment | padded B per segment | room past it for the GEMM's stream-K partials
  __nv_bfloat16* su[3] = {nullptr, nullptr, nullptr};
  __nv_bfloat16* bpad[3] = {nullptr, nullptr, nullptr};
  char* cur = static_cast<char*>(workspace);
  if (r > 0) {
    for (int i = 0; i < nseg; ++i, cur += f.su) su[i] = reinterpret_cast<__nv_bfloat16*>(cur);
    for (int i = 0; i < nseg; ++i) {
      bpad[i] = reinterpret_cast<__nv_bfloat16*>(cur);
      cur += f.bpad[i];
    }
  }
  char* sk_ws = nullptr;
  size_t sk_bytes = 0;
  if (workspace && aligned(workspace, 256) && workspace_bytes > base) {
    sk_ws = static_cast<char*>(workspace) + base;
    sk_bytes = workspace_bytes - base;
  }
  return tc::fwd_impl(nseg, W, x, M, A, B, r, s, residual, y, u_out, su, bpad, true, nullptr, nullptr, sk_ws,
                      sk_bytes, (cudaStream_t)stream, rope);
}

extern "C" size_t lsq_nf4_lora_state_size(int32_t nseg, int64_t M, int64_t k_in, const int64_t* n_out, int32_t r) {
  if (nseg < 1 || nseg > 3 || r <= 0 || r > 64 || M < 1 || k_in < 64 || !n_out) return 256;
  return lsq::tc::state_plan(nseg, M, k_in, n_out, r).total;
}

extern "C" lsq_status lsq_nf4_lora_fwd_multi_ex(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M,
                                                const void* const* A, const void* const* B, int32_t r, float s,
                                                const void* const* residual, void* const* y, float* const* u_out,
                                                void* state, int32_t state_ready, void* workspace,
                                                size_t workspace_bytes, lsq_cuda_stream stream) {
  using namespace lsq;
  const char* who = "lsq_nf4_lora_fwd_ex";
  int64_t ns[3];
  lsq_status st = tc::fwd_checks(nseg, W, x, M, A, B, r, residual, y, ns, who);
  if (st != LSQ_OK) return st;
  const int64_t K = W[0].k_in;
  if (r > 0 && (!state || !aligned(state, 256)))
    return fail(LSQ_EINVAL, "%s: a 256-byte aligned rank state is needed with r > 0", who);
  if (workspace && !aligned(workspace, 256)) return fail(LSQ_EINVAL, "%s: workspace must be 256-byte aligned", who);
  tc::StatePtrs q;
  memset(&q, 0, sizeof(q));
  if (r > 0) q = tc::state_ptrs(state, nseg, tc::state_plan(nseg, M, K, ns, r));
  return tc::fwd_impl(nseg, W, x, M, A, B, r, s, residual, y, u_out, q.su, q.bpad, !state_ready, q.bt, q.at,
                      static_cast<char*>(workspace), workspace ? workspace_bytes : 0, (cudaStream_t)stream);
}

extern "C" lsq_status lsq_nf4_lora_fwd_multi_ex2(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M,
                                                 const void* const* A, const void* const* B, int32_t r, float s,
                                                 const void* const* residual, void* const* y, float* const* u_out,
                                                 void* state, int32_t state_ready, const lsq_rope_spec* rope,
                                                 void* workspace, size_t workspace_bytes, lsq_cuda_stream stream) {
  using namespace lsq;
  const char* who = "lsq_nf4_lora_fwd_ex2";
  if (rope && rope->segments) {
    if (!rope->table || !aligned(rope->table, 16) || (rope->hd != 64 && rope->hd != 128 && rope->hd != 256) ||
        rope->seq < 1 || M % rope->seq != 0 || (rope->segments >> nseg) != 0)
      return fail(LSQ_EINVAL, "%s: RoPE needs a 16-byte aligned table, hd 64, 128 or 256, M a multiple of seq "
                  "and segment bits below nseg", who);
    for (int i = 0; i < nseg; ++i)
      if (((rope->segments >> i) & 1) && (!W || W[i].n_out % rope->hd != 0 || (residual && residual[i])))
        return fail(LSQ_EINVAL, "%s: a rotated segment needs n_out a multiple of hd and no residual", who);
  }
  if (!state)  // no rank state: the operands are rebuilt in the workspace, as lsq_nf4_lora_fwd_multi does
    return tc::fwd_multi_ws(nseg, W, x, M, A, B, r, s, residual, y, u_out, workspace, workspace_bytes, stream,
                            rope && rope->segments ? rope : nullptr, who);
  if (!rope || !rope->segments)
    return lsq_nf4_lora_fwd_multi_ex(nseg, W, x, M, A, B, r, s, residual, y, u_out, state, state_ready, workspace,
                                     workspace_bytes, stream);
  int64_t ns[3];
  lsq_status st = tc::fwd_checks(nseg, W, x, M, A, B, r, residual, y, ns, who);
  if (st != LSQ_OK) return st;
  const int64_t K = W[0].k_in;
  if (r > 0 && (!state || !aligned(state, 256)))
    return fail(LSQ_EINVAL, "%s: a 256-byte aligned rank state is needed with r > 0", who);
  if (workspace && !aligned(workspace, 256)) return fail(LSQ_EINVAL, "%s: workspace must be 256-byte aligned", who);
  tc::StatePtrs q;
  memset(&q, 0, sizeof(q));
  if (r > 0) q = tc::state_ptrs(state, nseg, tc::state_plan(nseg, M, K, ns, r));
  return tc::fwd_impl(nseg, W, x, M, A, B, r, s, residual, y, u_out, q.su, q.bpad, !state_ready, q.bt, q.at,
                      static_cast<char*>(workspace), workspace ? workspace_bytes : 0, (cudaStream_t)stream, rope);
}

extern "C" lsq_status lsq_nf4_lora_fwd(const lsq_nf4_weight* W, const void* x, int64_t M, const void* A,
                                       const void* B, int32_t r, float s, const void* residual, void* y,
                                       float* u_out, void* workspace, size_t workspace_bytes,
                                       lsq_cuda_stream stream) {
  const void* a[1] = {A};
  const void* b[1] = {B};
  const void* res[1] = {residual};
  void* yy[1] = {y};
  float* uu[1] = {u_out};
  return lsq_nf4_lora_fwd_multi(1, W, x, M, a, b, r, s, res, yy, uu, workspace, workspace_bytes, stream);
}
