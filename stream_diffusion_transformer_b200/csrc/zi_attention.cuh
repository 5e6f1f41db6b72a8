// Non-causal flash attention (head_dim 128, bf16 in/out, fp32 softmax) on tcgen05,
// one CTA pair (a cluster of 2 CTAs on two SMs) per pair of 128-query tiles.
//
// CTA r of the pair holds query tile 2u + r.  One thread of CTA 0 issues every
// tensor-core instruction for both SMs with tcgen05 cta_group::2 (M = 256, 128 rows
// per SM):
//   S = Q K^T    A = each CTA's Q tile in smem, B = the key tile, keys
//                [64 r, 64 r + 64) in CTA r's smem;
//   O += P V     A = each CTA's P in TMEM, B = the value tile, head dims
//                [64 r, 64 r + 64) in CTA r's smem.
// Each SM's 512 TMEM columns hold two S buffers [0, 256), O [256, 384) and two P
// buffers [384, 512) for its 128 rows, so nothing aliases: S_{j+2} is computed
// into S_j's buffer while PV_j runs, the two being issued interleaved in runs of
// four MMAs, and the softmax of tile j + 1 never waits for PV_j.  Per CTA, 12 warps
// (registers move to the softmax warps with setmaxnreg: launch 168 per thread,
// softmax 200, others 96):
//   warps 0..7  softmax: warps w and w + 4 share the 32 rows of TMEM lanes
//               32 (w mod 4) ..; warp w < 4 takes keys 0..63 of each tile (and
//               head dims 0..63 of O), warp w + 4 the rest.  The two halves of a
//               row exchange partial maxima through shared memory, so they keep
//               the same running max.  Online softmax in the exp2 domain with a
//               lazily updated running max (O rescaled in TMEM only when a row's
//               max grows by more than 2^8); P is stored to TMEM as bf16 pairs and
//               signalled to CTA 0's MMA thread (a remote mbarrier arrive from CTA 1)
//   warp 8      TMA: this CTA's Q tile, then its halves of the key and value tiles
//               through a 5-entry ring ({K_0, K_1}, then {V_j, K_{j+2}}), straight
//               out of the fused [rows, 3D] projection buffer; the copies of both
//               CTAs complete on CTA 0's barriers (TMA cta_group::2)
//   warp 9      TMEM allocation for the pair; in CTA 0 lane 0 issues the MMAs and
//               commits them to the barriers of both CTAs (multicast commit)
//   warps 10-11 idle
// The issuing thread shares its SM sub-partition with two busy softmax warps, so
// its per-MMA instruction count is kept small: operand descriptors are a base
// plus a constant per MMA, and accumulating MMAs use a constant predicate.
// The key sequence of a batch element can be split over two row segments of the
// token buffer (image rows and text rows); key tiles that run past a segment's
// end are masked to -inf.  An optional per-element key count for the last segment
// (kv_len) drops that segment's trailing rows (padding) from the keys: tiles
// wholly past it are never loaded, the tile it ends in is masked.
#pragma once
#include "zi_common.cuh"

namespace zi {

struct AttnParams {
  uint16_t* out;  // bf16 [rows, ldo]; head h at columns [h*128, h*128 + 128)
  int ldo;
  int dim;        // D: K block starts at column D of the projection buffer, V at 2D
  int nseg;       // 1 or 2
  int seg_row0[2];  // first row of segment i for batch element 0
  int seg_len[2];   // rows per batch element in segment i (element b starts at row0 + b * len)
  int q_tiles;      // query tiles per batch element (both segments)
  float scale_log2; // log2(e) / sqrt(head_dim)
  const int* kv_len;  // [batch] keys of the last segment per element, or null (= its seg_len)
  int heads;          // units are (pair of query tiles, head, batch element), pair fastest
};

// Keys of the last segment of element b: kv_len[b] clamped to [1, seg_len], or all.
ZI_DEV int attn_last_len(const AttnParams& p) { return p.nseg > 1 ? p.seg_len[1] : p.seg_len[0]; }

ZI_DEV int attn_last_keys(const AttnParams& p, int b) {
  const int n = attn_last_len(p);
  if (!p.kv_len) return n;
  return max(1, min(n, p.kv_len[b]));
}

// Rows of tile `tile` of element b; the last segment counts last_n rows (all of
// them for query tiles, the element's key count for key tiles).
ZI_DEV void attn_tile_rows(const AttnParams& p, int b, int tile, int last_n, int& row0, int& valid) {
  int seg = 0;
  int t = tile;
  const int n0 = (p.seg_len[0] + 127) / 128;
  if (p.nseg > 1 && t >= n0) {
    seg = 1;
    t -= n0;
  }
  // seg is 0 or 1: select rather than index, so the parameters stay in constant space
  const int row0_s = seg ? p.seg_row0[1] : p.seg_row0[0];
  const int len_s = seg ? p.seg_len[1] : p.seg_len[0];
  row0 = row0_s + b * len_s + t * 128;
  valid = min(128, (seg == p.nseg - 1 ? last_n : len_s) - t * 128);
}

ZI_DEV float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Packed fp32 pair arithmetic (one instruction for two values).
ZI_DEV uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
ZI_DEV void f2_unpack(uint64_t v, float& lo, float& hi) { asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v)); }
ZI_DEV uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
ZI_DEV uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
ZI_DEV uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// 2^x for a pair on the FMA pipe (FlashAttention-4's relief for the 16/clk/SM
// MUFU): Cody-Waite split x = n + f with n = rint(x) (the 1.5 * 2^23 rounding
// trick), f in [-1/2, 1/2]; 2^f by a degree-3 polynomial whose coefficients were
// fitted here by the Remez exchange algorithm on the relative error (max
// relative error 7.5e-5, far below the bf16 rounding P gets next); n is added
// to the exponent field.  x is clamped at -126 so the result stays normal.
ZI_DEV void exp2_poly_pair(float x0, float x1, float& e0, float& e1) {
  x0 = fmaxf(x0, -126.0f);
  x1 = fmaxf(x1, -126.0f);
  const uint64_t x2 = f2_pack(x0, x1);
  const uint64_t t2 = f2_add(x2, f2_pack(12582912.0f, 12582912.0f));
  const uint64_t n2 = f2_add(t2, f2_pack(-12582912.0f, -12582912.0f));
  const uint64_t fr = f2_fma(n2, f2_pack(-1.0f, -1.0f), x2);
  uint64_t p2 = f2_fma(f2_pack(0.05517166853f, 0.05517166853f), fr, f2_pack(0.2426111251f, 0.2426111251f));
  p2 = f2_fma(p2, fr, f2_pack(0.6932609677f, 0.6932609677f));
  p2 = f2_fma(p2, fr, f2_pack(0.9999280572f, 0.9999280572f));
  float t0, t1, p0, p1;
  f2_unpack(t2, t0, t1);
  f2_unpack(p2, p0, p1);
  e0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  e1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

namespace attn {
constexpr int kThreads = 384;
constexpr int kRegsSoftmax = 200;  // 2 x 128 x 200 + 128 x 96 = 63488 <= 384 x 168 registers at launch
constexpr int kRegsOther = 96;
constexpr uint32_t kHalfTile = 64 * 128 * 2;   // 16 KB: K half (64 keys x 128 dims) or V half (128 keys x 64 dims)
constexpr uint32_t kKBox = 64 * 64 * 2;        // 8 KB: 64 keys x 64 dims (one swizzled box of a K half)
constexpr int kEntries = 5;                    // ring entries of 2 half tiles
constexpr uint32_t kQ0 = 0;                    // Q tile, two 64-dim halves of 16 KB
constexpr uint32_t kR0 = 32768;
constexpr uint32_t kXch = kR0 + kEntries * 2 * kHalfTile;  // [2 parities][2 halves][128 rows] fp32
constexpr uint32_t kBar = kXch + 2 * 2 * 128 * 4;
constexpr uint32_t kSmemBytes = kBar + 256 + 1024;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;  // S_j at 128 (j mod 2), P_j at kColP + 64 (j mod 2)
}  // namespace attn

ZI_DEV uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
ZI_DEV void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory offset in CTA 0 of the pair (shared::cluster window).
ZI_DEV uint32_t leader_addr(const void* ptr) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(smem_u32(ptr)));
  return r;
}
// Arrive once on the barrier at the same shared-memory offset in CTA 0 of the pair.
ZI_DEV void mbar_arrive_leader(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(leader_addr(bar)) : "memory");
}
// TMA load into this CTA's shared memory whose bytes complete on CTA 0's barrier.
ZI_DEV void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_addr(bar)), "r"(x), "r"(y)
      : "memory");
}
// tcgen05.mma cta_group::2 (M = 256 over the pair), D (+)= A * B: A in smem (ss) or TMEM
// (ts).  The _acc forms always accumulate, with a constant predicate.
ZI_DEV void tc_mma2_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
ZI_DEV void tc_mma2_ss_acc(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.eq.u32 p, 1, 1;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc)
      : "memory");
}
ZI_DEV void tc_mma2_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
ZI_DEV void tc_mma2_ts_acc(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.eq.u32 p, 1, 1;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc)
      : "memory");
}
// Arrive on the barrier at this offset in both CTAs of the pair when the MMAs issued so far complete.
ZI_DEV void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(uint16_t(3))
      : "memory");
}

// The kernel (see the file comment).  Grid: 2 CTAs per unit, cluster dims 2.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(attn::kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     AttnParams p) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* xch = reinterpret_cast<float*>(smem + kXch);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBar);
  uint64_t* q_full = bars + 0;     // CTA 0: both Q tiles loaded
  uint64_t* r_full = bars + 1;     // [kEntries] CTA 0: both CTAs' halves of the entry loaded
  uint64_t* r_empty = bars + 6;    // [kEntries] each CTA: entry released by its last MMA
  uint64_t* s_full = bars + 11;    // [2] each CTA: S buffer computed
  uint64_t* p_full = bars + 13;    // [2] CTA 0: P buffer stored by both CTAs' softmax threads
  uint64_t* pv_done = bars + 15;   // [2] each CTA: the PV that read P buffer b complete
  uint64_t* xbar = bars + 17;      // [4 lane quadrants] row-half exchange
  uint64_t* drain = bars + 21;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 22);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int unit = blockIdx.x >> 1;
  const int pairs = (p.q_tiles + 1) >> 1;
  const int pair = unit % pairs, head = (unit / pairs) % p.heads, b = unit / (pairs * p.heads);
  const int last_keys = attn_last_keys(p, b);
  const int nj = p.nseg > 1 ? (p.seg_len[0] + 127) / 128 + (last_keys + 127) / 128 : (last_keys + 127) / 128;
  const int my_tile = 2 * pair + int(rank);
  const bool has_tile = my_tile < p.q_tiles;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kEntries; ++i) {
      mbar_init(&r_full[i], 1);
      mbar_init(&r_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 512);
      mbar_init(&pv_done[i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&xbar[i], 64);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated before any remote access
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool err = device_error_set();
  const int colq = head * 128, colk = p.dim + head * 128, colv = 2 * p.dim + head * 128;

  if (!err && warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
   if (warp == 8) {
    if (lane == 0) {
      // Q of this CTA's tile (the last pair may hold one tile: its partner loads the same rows)
      int q0, qv;
      attn_tile_rows(p, b, has_tile ? my_tile : my_tile - 1, attn_last_len(p), q0, qv);
      if (rank == 0) mbar_arrive_expect_tx(q_full, 2 * 32768);
      tma_load_2d_pair(smem + kQ0, &tm_q, q_full, colq, q0);
      tma_load_2d_pair(smem + kQ0 + 16384, &tm_q, q_full, colq + 64, q0);
      // ring entry e: e = 0 holds K_0 and K_1 halves, e = j + 1 the V_j half and the K_{j+2} half
      for (int e = 0; e <= nj; ++e) {
        const int slot = e % kEntries;
        const uint32_t r = uint32_t(e / kEntries);
        const int m0 = e == 0 ? 0 : e - 1, m1 = e == 0 ? 1 : e + 1;
        const bool has1 = m1 < nj;
        if (!mbar_wait(&r_empty[slot], (r & 1u) ^ 1u, abort_flag, ZI_DEVERR_TIMEOUT_PRODUCER)) break;
        uint8_t* dst = smem + kR0 + slot * 2 * kHalfTile;
        if (rank == 0) mbar_arrive_expect_tx(&r_full[slot], (has1 ? 2u : 1u) * 2u * kHalfTile);
        int kv0, kvn;
        attn_tile_rows(p, b, m0, last_keys, kv0, kvn);
        if (e == 0) {  // K_0 half: keys [64 r, 64 r + 64), both 64-dim boxes
          tma_load_2d_pair(dst, &tm_k, &r_full[slot], colk, kv0 + 64 * int(rank));
          tma_load_2d_pair(dst + kKBox, &tm_k, &r_full[slot], colk + 64, kv0 + 64 * int(rank));
        } else {       // V_j half: all 128 keys, head dims [64 r, 64 r + 64)
          tma_load_2d_pair(dst, &tm_q, &r_full[slot], colv + 64 * int(rank), kv0);
        }
        if (has1) {
          attn_tile_rows(p, b, m1, last_keys, kv0, kvn);
          tma_load_2d_pair(dst + kHalfTile, &tm_k, &r_full[slot], colk, kv0 + 64 * int(rank));
          tma_load_2d_pair(dst + kHalfTile + kKBox, &tm_k, &r_full[slot], colk + 64, kv0 + 64 * int(rank));
        }
      }
    }
   } else if (warp == 9) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(256, 128, false, false);  // B = K half, K-major
      constexpr uint32_t idesc_o = idesc_bf16_f32(256, 128, false, true);   // B = V half, MN-major
      // descriptors: a base per operand, plus each MMA's byte offset / 16 (a constant),
      // so the issuing thread spends few instructions per MMA
      const uint64_t desc_q = smem_desc_sw128(smem_u32(smem + kQ0), 16);
      const uint32_t ring0 = smem_u32(smem + kR0);
      const uint64_t desc_k0 = smem_desc_sw128(ring0, 16), desc_v0 = smem_desc_sw128(ring0, 8192);
      const uint32_t t_s0 = tmem + kColS, t_o = tmem + kColO, t_p0 = tmem + kColP;
      auto s_mma = [&](uint32_t ds, uint64_t kdesc, int k) {
        const uint64_t ad = desc_q + uint64_t(((k >> 2) * 16384 + (k & 3) * 32) >> 4);
        const uint64_t bd = kdesc + uint64_t(((k >> 2) * kKBox + (k & 3) * 32) >> 4);
        if (k == 0) tc_mma2_ss(ds, ad, bd, idesc_s, 0u);
        else tc_mma2_ss_acc(ds, ad, bd, idesc_s);
      };
      auto pv_mma = [&](uint32_t tp, uint64_t vdesc, int k, uint32_t acc) {
        if (k == 0) tc_mma2_ts(t_o, tp, vdesc, idesc_o, acc);
        else tc_mma2_ts_acc(t_o, tp + 8 * k, vdesc + uint64_t(k * 128), idesc_o);
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, ZI_DEVERR_TIMEOUT_MMA) &&
                mbar_wait(&r_full[0], 0, abort_flag, ZI_DEVERR_TIMEOUT_MMA);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k) s_mma(t_s0, desc_k0, k);
        tc_commit_pair(&s_full[0]);
        if (nj > 1) {
#pragma unroll
          for (int k = 0; k < 8; ++k) s_mma(t_s0 + 128, desc_k0 + (kHalfTile >> 4), k);
          tc_commit_pair(&s_full[1]);
        }
        tc_commit_pair(&r_empty[0]);
      }
      for (int j = 0; j < nj && ok; ++j) {
        const int e = j + 1, slot = e % kEntries;
        ok = mbar_wait(&p_full[j & 1], uint32_t(j >> 1) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA) &&
             mbar_wait(&r_full[slot], uint32_t(e / kEntries) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA);
        if (!ok) break;
        tc_fence_after();
        const uint64_t vdesc = desc_v0 + uint64_t(slot * (2 * kHalfTile >> 4));
        const uint64_t kdesc = desc_k0 + uint64_t(slot * (2 * kHalfTile >> 4) + (kHalfTile >> 4));
        const uint32_t ds = t_s0 + 128 * (j & 1), tp = t_p0 + 64 * (j & 1);
        const bool s_next = j + 2 < nj;
        // PV_j 0-3, S_{j+2} 0-3, PV_j 4-7 (signalled), S_{j+2} 4-7
        pv_mma(tp, vdesc, 0, j > 0 ? 1u : 0u);
#pragma unroll
        for (int k = 1; k < 4; ++k) pv_mma(tp, vdesc, k, 1u);
        if (s_next) {
#pragma unroll
          for (int k = 0; k < 4; ++k) s_mma(ds, kdesc, k);
        }
#pragma unroll
        for (int k = 4; k < 8; ++k) pv_mma(tp, vdesc, k, 1u);
        tc_commit_pair(&pv_done[j & 1]);
        if (s_next) {
#pragma unroll
          for (int k = 4; k < 8; ++k) s_mma(ds, kdesc, k);
          tc_commit_pair(&s_full[j & 1]);
        }
        tc_commit_pair(&r_empty[slot]);
      }
      if (!ok) {
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(drain))
                     : "memory");
        volatile int never = 0;
        mbar_wait(drain, 0, &never, ZI_DEVERR_TIMEOUT_DRAIN);
      }
    }
   }
  } else if (!err) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int h = warp >> 2;        // key half (and O head-dim half) of the row
    const int q = warp & 3;
    const int i = q * 32 + lane;    // query row in the tile == TMEM lane
    int q_row0, q_valid;
    attn_tile_rows(p, b, has_tile ? my_tile : my_tile - 1, attn_last_len(p), q_row0, q_valid);
    const uint32_t lane_addr = tmem + (uint32_t(q * 32) << 16);
    const uint32_t o_addr = lane_addr + kColO + 64 * h;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l = 0.f;
    uint32_t s[64];
    bool ok = true;
    for (int j = 0; j < nj; ++j) {
      int kv0, kvn;
      attn_tile_rows(p, b, j, last_keys, kv0, kvn);
      if (!mbar_wait(&s_full[j & 1], uint32_t(j >> 1) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_addr = lane_addr + kColS + 128 * (j & 1) + 64 * h;
      tmem_ld32(s_addr, &s[0]);
      tmem_ld32(s_addr + 32, &s[32]);
      tmem_wait_ld();
      reg_fence32(&s[0]);
      reg_fence32(&s[32]);
      if (kvn < 128) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (64 * h + c >= kvn) s[c] = __float_as_uint(-INFINITY);
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = max3f(__uint_as_float(s[k]), __uint_as_float(s[8 + k]), __uint_as_float(s[16 + k]));
#pragma unroll
      for (int c = 24; c < 56; c += 16) {
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = max3f(mx8[k], __uint_as_float(s[c + k]), __uint_as_float(s[c + 8 + k]));
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(mx8[k], __uint_as_float(s[56 + k]));
      const float pm = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
      xch[(j & 1) * 256 + h * 128 + i] = pm;
      mbar_arrive(&xbar[q]);
      if (!mbar_wait(&xbar[q], uint32_t(j) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX)) { ok = false; break; }
      const float mx = fmaxf(pm, xch[(j & 1) * 256 + (h ^ 1) * 128 + i]);
      const float m_new = fmaxf(m_run, mx * sl2);
      const bool resc = __any_sync(0xffffffffu, m_new > m_run + 8.0f);
      float alpha = 1.0f;
      if (resc) {
        alpha = fast_exp2(m_run - m_new);
        m_run = m_new;
        l *= alpha;
      }
      const uint64_t sl2x2 = f2_pack(sl2, sl2), negm = f2_pack(-m_run, -m_run);
      uint64_t sum2[4] = {0, 0, 0, 0};
      uint32_t pw[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), sl2x2, negm), x0, x1);
        float e0, e1;
        if ((c & 7) == 4) {  // 1 of 8 pairs on the FMA pipe (fewer issue slots taken from the MMA thread)
          exp2_poly_pair(x0, x1, e0, e1);
        } else {
          e0 = fast_exp2(x0);
          e1 = fast_exp2(x1);
        }
        sum2[c & 3] = f2_add(sum2[c & 3], f2_pack(e0, e1));
        pw[c] = pack_bf16x2(e0, e1);
      }
      {
        float a0, a1, b0, b1, c0, c1, d0, d1;
        f2_unpack(sum2[0], a0, a1);
        f2_unpack(sum2[1], b0, b1);
        f2_unpack(sum2[2], c0, c1);
        f2_unpack(sum2[3], d0, d1);
        l += ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
      }
      // P buffer j mod 2 is free once PV_{j-2} completed; a rescale needs PV_{j-1} in O
      if (j >= 2 && !mbar_wait(&pv_done[j & 1], uint32_t((j - 2) >> 1) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX)) {
        ok = false;
        break;
      }
      if (resc && j > 0) {
        if (!mbar_wait(&pv_done[(j - 1) & 1], uint32_t((j - 1) >> 1) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          tmem_ld32_sync(o_addr + c * 32, o);
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            float y0, y1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(o[2 * k]), __uint_as_float(o[2 * k + 1])), a2), y0, y1);
            o[2 * k] = __float_as_uint(y0);
            o[2 * k + 1] = __float_as_uint(y1);
          }
          tmem_st32(o_addr + c * 32, o);
        }
      } else if (j >= 2) {
        tc_fence_after();
      }
      tmem_st32(lane_addr + kColP + 64 * (j & 1) + 32 * h, pw);
      tmem_wait_st();
      tc_fence_before();
      if (rank == 0) mbar_arrive(&p_full[j & 1]);
      else mbar_arrive_leader(&p_full[j & 1]);
    }
    ok = ok && mbar_wait(&pv_done[(nj - 1) & 1], uint32_t((nj - 1) >> 1) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX);
    if (ok) {
      tc_fence_after();
      xch[(nj & 1) * 256 + h * 128 + i] = l;
      mbar_arrive(&xbar[q]);
      ok = mbar_wait(&xbar[q], uint32_t(nj) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX);
      if (ok) l += xch[(nj & 1) * 256 + (h ^ 1) * 128 + i];
    }
    if (ok && has_tile) {
      const float inv = 1.0f / l;
      uint16_t* orow = p.out + size_t(q_row0 + i) * p.ldo + head * 128 + 64 * h;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tmem_ld32_sync(o_addr + c * 32, o);
        if (i < q_valid) {
          uint4* d = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * k + 0]) * inv, __uint_as_float(o[8 * k + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * k + 2]) * inv, __uint_as_float(o[8 * k + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * k + 4]) * inv, __uint_as_float(o[8 * k + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * k + 6]) * inv, __uint_as_float(o[8 * k + 7]) * inv);
            d[k] = w;
          }
        }
      }
    }
  }

  if (*abort_flag) {  // an aborted pipeline: let copies already issued land before the pair leaves
    const unsigned long long t0 = globaltimer();
    while (globaltimer() - t0 < 200000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA frees TMEM or exits while the pair's MMAs or copies may use it
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
  }
}

}  // namespace zi
