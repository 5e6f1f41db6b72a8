// Non-causal flash attention (head_dim 128, bf16 in/out, fp32 softmax) on tcgen05.
//
// One CTA per (pair of 128-query tiles A and B, head, batch element), 12 warps
// in three warpgroups; registers move from the third to the first two with
// setmaxnreg (launch 168 per thread; softmax 216, TMA/MMA 56):
//   warp 8      TMA: both Q tiles once, then K tiles (128 keys each) into a
//               3-deep ring, straight out of the fused [rows, 3D] projection
//               buffer (the head's 128 columns as two 64-wide swizzled boxes)
//   warp 9      TMEM allocator + tcgen05.mma issuer.  TMEM: S_A, S_B, O_A, O_B,
//               128 columns each.  Per key tile j the tensor core runs
//                 S_A(j+1) = Q_A K^T, O_B += P_B(j) V, S_B(j+1) = Q_B K^T, O_A += P_A(j+1) V
//               so each tile's softmax has the other tile's two MMAs to hide behind.
//   warp 10     TMA for the 2-deep V ring (warp 8 then only loads Q and K)
//   warp 11     idle
//   warps 0..3  softmax of tile A, warps 4..7 softmax of tile B: one thread per
//               query row (its TMEM lane); online softmax in the exp2 domain with a
//               lazily updated running max (O rescaled in TMEM only when a row's max
//               grows by more than 2^8); P (bf16) is written back over the first 64
//               columns of its S and read from TMEM by the PV MMA.
// A tcgen05.mma that overwrites S(j+1) is issued after the MMA that reads P(j)
// from the same columns; the tensor core executes one CTA's MMAs in issue order.
// The key sequence of a batch element can be split over two row segments of
// the token buffer (image rows and text rows); key tiles that run past a
// segment's end are masked to -inf.  An optional per-element key count for the
// last segment (kv_len) drops that segment's trailing rows (padding) from the
// keys: tiles wholly past it are never loaded, the tile it ends in is masked.
//
// Work units are (query-tile pair, head, batch element), one CTA each.  When the
// units leave a ragged last wave of R < G (SM count) units and scratch is given,
// those R units are cut along the keys into s pieces (s R <= G), one CTA per
// piece: each piece writes its unnormalised O rows with their running max and
// sum, and the piece that completes the unit's counter merges the pieces in
// piece order (the same order whichever piece finishes) and writes the output.
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
  int pairs, heads;   // units are (pair of query tiles, head, batch element), pair fastest
  int full_units;     // units [0, full_units) run whole, one CTA each
  int split_s;        // key pieces per remaining unit (1 = none)
  float4* part;       // split scratch: kAttnSlotF4 float4 per piece (null = no split)
  int* counters;      // one per split unit, zero on entry (the finisher resets it)
};

namespace attn {
constexpr int kThreads = 384;
constexpr int kRegsSoftmax = 216;  // 2 x 128 x 216 + 128 x 56 = 62464 <= 384 x 168 registers at launch
constexpr int kRegsOther = 56;
constexpr uint32_t kTile = 128 * 128 * 2;  // one 128 x 128 bf16 tile (two 64-column halves)
constexpr uint32_t kHalf = kTile / 2;
constexpr int kKSlots = 3, kVSlots = 2;  // K ring one deeper than V (smem holds 7 tiles)
constexpr uint32_t kQ0 = 0, kK0 = 2 * kTile, kV0 = kK0 + kKSlots * kTile;
constexpr uint32_t kBar = kV0 + kVSlots * kTile;
constexpr uint32_t kSmemBytes = kBar + 256 + 1024;
constexpr uint32_t kColS = 0, kColO = 256;  // S_t at kColS + 128 t, O_t at kColO + 128 t
constexpr int kMaxSplit = 4;
// one piece's partial: O of both tiles [t][32 column quads][128 rows] float4, then
// (m, l) of both tiles [t][128 rows] float2
constexpr int kSlotOF4 = 2 * 32 * 128;
constexpr int kSlotF4 = kSlotOF4 + 128;
}  // namespace attn

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

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16, A (bf16) read from TMEM.
ZI_DEV void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
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
// relative error 7.5e-5 on [-125, 0], far below the bf16 rounding P gets next); n
// is added to the exponent field.  x is clamped at -126; below -125 the result may
// be denormal and is at most 2^-124 (zero at P's precision against a row max of 1).
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

__global__ void __launch_bounds__(attn::kThreads, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm, AttnParams p) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [kKSlots]
  uint64_t* k_empty = bars + 4;   // [kKSlots]
  uint64_t* v_full = bars + 7;    // [kVSlots]
  uint64_t* v_empty = bars + 9;   // [kVSlots]
  uint64_t* s_full = bars + 11;   // [2 tiles]
  uint64_t* p_full = bars + 13;   // [2 tiles]
  uint64_t* pv_done = bars + 15;  // [2 tiles]
  uint64_t* drain = bars + 17;
  uint64_t* fin_bar = bars + 18;  // the softmax threads' meeting point (split pieces)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* fin_flag = abort_flag + 1;

  if (device_error_set()) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // which unit, and which piece of its keys, this CTA runs
  int unit = blockIdx.x, piece = -1;
  if (unit >= p.full_units) {
    const int v = unit - p.full_units;
    unit = p.full_units + v / p.split_s;
    piece = v % p.split_s;
  }
  const int pair = unit % p.pairs, head = (unit / p.pairs) % p.heads, b = unit / (p.pairs * p.heads);
  const int last_keys = attn_last_keys(p, b);
  const int n_kv = p.nseg > 1 ? (p.seg_len[0] + 127) / 128 + (last_keys + 127) / 128 : (last_keys + 127) / 128;
  // key tiles [j0, j0 + nj) of this CTA (all of them for a whole unit)
  const int j0 = piece < 0 ? 0 : piece * n_kv / p.split_s;
  const int nj = piece < 0 ? n_kv : (piece + 1) * n_kv / p.split_s - j0;
  const int tile_a = 2 * pair;
  const bool has_b = tile_a + 1 < p.q_tiles;  // CTA-uniform: the last pair may hold one tile

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kKSlots; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kVSlots; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);  // one arrival per softmax warp
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain, 1);
    mbar_init(fin_bar, has_b ? 256 : 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) prefetch_tmap(&tm);
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int colq = head * 128, colk = p.dim + head * 128, colv = 2 * p.dim + head * 128;

  // Each role's code sits inside the branch that set its register budget, so the
  // register allocator sees the budget that holds for it.
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
   if (warp == 8 || warp == 10) {
    // warp 8 loads Q and the K ring, warp 10 the V ring, so neither ring's wait
    // holds up the other's next load
    if (lane == 0) {
      const bool kq = warp == 8;
      if (kq) {
        int qa0, qav, qb0 = 0, qbv = 0;
        attn_tile_rows(p, b, tile_a, attn_last_len(p), qa0, qav);
        if (has_b) attn_tile_rows(p, b, tile_a + 1, attn_last_len(p), qb0, qbv);
        mbar_arrive_expect_tx(q_full, has_b ? 2 * kTile : kTile);
        tma_load_2d(smem + kQ0, &tm, q_full, colq, qa0);
        tma_load_2d(smem + kQ0 + kHalf, &tm, q_full, colq + 64, qa0);
        if (has_b) {
          tma_load_2d(smem + kQ0 + kTile, &tm, q_full, colq, qb0);
          tma_load_2d(smem + kQ0 + kTile + kHalf, &tm, q_full, colq + 64, qb0);
        }
      }
      uint64_t* fullb = kq ? k_full : v_full;
      uint64_t* emptyb = kq ? k_empty : v_empty;
      const uint32_t base = kq ? kK0 : kV0;
      const int col = kq ? colk : colv;
      const int nslots = kq ? kKSlots : kVSlots;
      uint32_t issued = 0;
      bool ok = true;
      for (int j = 0; j < nj; ++j) {
        const int bi = j % nslots;
        const uint32_t r = uint32_t(j / nslots);
        int kv0, kvn;
        attn_tile_rows(p, b, j0 + j, last_keys, kv0, kvn);
        if (!mbar_wait(&emptyb[bi], (r & 1u) ^ 1u, abort_flag, ZI_DEVERR_TIMEOUT_PRODUCER)) { ok = false; break; }
        mbar_arrive_expect_tx(&fullb[bi], kTile);
        tma_load_2d(smem + base + bi * kTile, &tm, &fullb[bi], col, kv0);
        tma_load_2d(smem + base + bi * kTile + kHalf, &tm, &fullb[bi], col + 64, kv0);
        ++issued;
      }
      if (!ok) {
        volatile int never = 0;
        if (kq) mbar_wait(q_full, 0, &never, ZI_DEVERR_TIMEOUT_DRAIN);
        for (uint32_t j = (issued > uint32_t(nslots) ? issued - nslots : 0); j < issued; ++j)
          mbar_wait(&fullb[j % nslots], (j / nslots) & 1u, &never, ZI_DEVERR_TIMEOUT_DRAIN);
      }
    }
   } else if (warp == 9) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, false, true);
      const int ntile = has_b ? 2 : 1;
      bool ok = mbar_wait(q_full, 0, abort_flag, ZI_DEVERR_TIMEOUT_MMA);
      tc_fence_after();
      // S_t(j) = Q_t K_j^T into S_t
      auto issue_s = [&](int t, int j) {
        const uint32_t q_addr = smem_u32(smem + kQ0 + t * kTile);
        const uint32_t k_addr = smem_u32(smem + kK0 + (j % kKSlots) * kTile);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = smem_desc_sw128(q_addr + (k >> 2) * kHalf + (k & 3) * 32, 16);
          const uint64_t bd = smem_desc_sw128(k_addr + (k >> 2) * kHalf + (k & 3) * 32, 16);
          tc_mma(tmem + kColS + 128 * t, ad, bd, idesc_s, k > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[t]);
      };
      // O_t += P_t(j) V_j, P_t (bf16, 64 columns) read from the front of S_t
      auto issue_pv = [&](int t, int j) -> bool {
        if (!mbar_wait(&p_full[t], uint32_t(j) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + kV0 + (j & 1) * kTile);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t bd = smem_desc_sw128(v_addr + k * 2048, kHalf);
          tc_mma_ts(tmem + kColO + 128 * t, tmem + kColS + 128 * t + 8 * k, bd, idesc_o,
                    (j > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(&pv_done[t]);
        return true;
      };
      auto wait_k = [&](int j) {
        return mbar_wait(&k_full[j % kKSlots], uint32_t(j / kKSlots) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA);
      };
      auto wait_v = [&](int j) {
        return mbar_wait(&v_full[j & 1], (uint32_t(j) >> 1) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA);
      };
      // prologue: S_A(0), S_B(0), O_A += P_A(0) V_0
      if (ok && wait_k(0)) {
        tc_fence_after();
        issue_s(0, 0);
        if (ntile > 1) issue_s(1, 0);
        tc_commit(&k_empty[0]);
        ok = wait_v(0) && issue_pv(0, 0);
      } else {
        ok = false;
      }
      for (int j = 0; j < nj && ok; ++j) {
        const bool more = j + 1 < nj;
        if (more) {
          if (!wait_k(j + 1)) { ok = false; break; }
          tc_fence_after();
          issue_s(0, j + 1);
        }
        if (ntile > 1 && !issue_pv(1, j)) { ok = false; break; }
        tc_commit(&v_empty[j & 1]);
        if (more) {
          if (ntile > 1) issue_s(1, j + 1);
          tc_commit(&k_empty[(j + 1) % kKSlots]);
          if (!wait_v(j + 1) || !issue_pv(0, j + 1)) { ok = false; break; }
        }
      }
      if (!ok) {
        tc_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, ZI_DEVERR_TIMEOUT_DRAIN);
      }
    }
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // softmax warpgroups: t = 0 (warps 0..3) handles tile A, t = 1 (warps 4..7) tile B
    const int t = warp >> 2;
    const int q = warp & 3;
    const int i = q * 32 + lane;  // query row in the tile == TMEM lane
    if (t == 0 || has_b) {
      int q_row0, q_valid;
      attn_tile_rows(p, b, tile_a + t, attn_last_len(p), q_row0, q_valid);
      const uint32_t lane_addr = tmem + (uint32_t(q * 32) << 16);
      const uint32_t s_addr = lane_addr + kColS + 128 * t;
      const uint32_t o_addr = lane_addr + kColO + 128 * t;
      const float sl2 = p.scale_log2;
      float m_run = -INFINITY, l = 0.f;
      uint32_t s[128];
      bool ok = true;
      for (int j = 0; j < nj; ++j) {
        int kv0, kvn;
        attn_tile_rows(p, b, j0 + j, last_keys, kv0, kvn);
        if (!mbar_wait(&s_full[t], uint32_t(j) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, &s[c * 32]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) reg_fence32(&s[c * 32]);
        if (kvn < 128) {  // the segment's last key tile: mask the columns past its end
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= kvn) s[c] = __float_as_uint(-INFINITY);
        }
        // row max: 3-input max over 8 independent chains
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = __uint_as_float(s[k]);
#pragma unroll
        for (int c = 8; c < 120; c += 16) {
#pragma unroll
          for (int k = 0; k < 8; ++k) mx8[k] = max3f(mx8[k], __uint_as_float(s[c + k]), __uint_as_float(s[c + 8 + k]));
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(mx8[k], __uint_as_float(s[120 + k]));
        const float mx = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool resc = __any_sync(0xffffffffu, m_new > m_run + 8.0f);
        float alpha = 1.0f;
        if (resc) {
          alpha = fast_exp2(m_run - m_new);
          m_run = m_new;
          l *= alpha;
        }
        // p = 2^(s * sl2 - m): packed FMA, exp2 on MUFU (5 of 8 pairs) or the FMA
        // pipe (3 of 8), packed row sums, bf16 pairs
        const uint64_t sl2x2 = f2_pack(sl2, sl2), negm = f2_pack(-m_run, -m_run);
        uint64_t sum2[4] = {0, 0, 0, 0};
        uint32_t pw[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), sl2x2, negm), x0, x1);
          float e0, e1;
          if ((c & 7) == 1 || (c & 7) == 4 || (c & 7) == 6) {  // 3 of 8 pairs on the FMA pipe
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
        if (resc && j > 0) {
          // O_t holds PV up to tile j-1: wait for that MMA, then scale O_t by alpha
          if (!mbar_wait(&pv_done[t], uint32_t(j - 1) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
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
        }
        // P over the first 64 columns of S_t (S_t(j) is already in registers)
        tmem_st32(s_addr, &pw[0]);
        tmem_st32(s_addr + 32, &pw[32]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[t]);  // for the whole warp: its stores are complete
      }
      ok = ok && mbar_wait(&pv_done[t], uint32_t(nj - 1) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX);
      if (ok) tc_fence_after();
      bool write = ok;
      // merged output of a split unit: O = sum_k 2^(m_k - M) O_k, l = sum_k 2^(m_k - M) l_k
      float mk[kMaxSplit], wk[kMaxSplit];
      float inv = 1.0f;
      const float4* slot0 = nullptr;
      if (ok && piece >= 0) {
        const int first = (unit - p.full_units) * p.split_s;  // slot of piece 0
        slot0 = p.part + size_t(first) * kSlotF4;
        float4* mine = p.part + size_t(first + piece) * kSlotF4;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32_sync(o_addr + c * 32, o);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            __stcg(mine + (t * 32 + c * 8 + k) * 128 + i,
                   make_float4(__uint_as_float(o[4 * k]), __uint_as_float(o[4 * k + 1]),
                               __uint_as_float(o[4 * k + 2]), __uint_as_float(o[4 * k + 3])));
        }
        __stcg(reinterpret_cast<float2*>(mine + kSlotOF4) + t * 128 + i, make_float2(m_run, l));
        __threadfence();
        mbar_arrive(fin_bar);
        ok = mbar_wait(fin_bar, 0, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX);
        if (ok && threadIdx.x == 0) {
          const int u = unit - p.full_units;
          const bool last = atomicAdd(&p.counters[u], 1) == p.split_s - 1;
          if (last) p.counters[u] = 0;  // ready for the next launch
          *fin_flag = last ? 1 : 0;
        }
        if (ok) {
          mbar_arrive(fin_bar);
          ok = mbar_wait(fin_bar, 1, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX);
        }
        write = ok && *fin_flag != 0;
        if (write) {
          __threadfence();
          float M = -INFINITY, L = 0.f;
#pragma unroll
          for (int k = 0; k < kMaxSplit; ++k) {
            mk[k] = -INFINITY;
            float lk = 0.f;
            if (k < p.split_s) {
              if (k == piece) {
                mk[k] = m_run;
                lk = l;
              } else {
                const float2 ml = __ldcg(reinterpret_cast<const float2*>(slot0 + size_t(k) * kSlotF4 + kSlotOF4) +
                                         t * 128 + i);
                mk[k] = ml.x;
                lk = ml.y;
              }
            }
            M = fmaxf(M, mk[k]);
            wk[k] = lk;  // l_k for now
          }
#pragma unroll
          for (int k = 0; k < kMaxSplit; ++k) {
            const float lk = wk[k];
            wk[k] = k < p.split_s ? fast_exp2(mk[k] - M) : 0.f;
            if (k < p.split_s) L = k == 0 ? wk[k] * lk : fmaf(wk[k], lk, L);
          }
          inv = 1.0f / L;
        }
      } else if (ok) {
        inv = 1.0f / l;
      }
      if (write) {
        uint16_t* orow = p.out + size_t(q_row0 + i) * p.ldo + head * 128;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32_sync(o_addr + c * 32, o);
          if (piece >= 0) {
            // the other pieces' 32 columns, loaded together before any is used
            float4 pp[kMaxSplit][8];
#pragma unroll
            for (int k = 0; k < kMaxSplit; ++k) {
              const bool need = k < p.split_s && k != piece;
              const float4* src = slot0 + size_t(k) * kSlotF4 + (t * 32 + c * 8) * 128 + i;
#pragma unroll
              for (int e = 0; e < 8; ++e) pp[k][e] = need ? __ldcg(src + e * 128) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
              for (int k = 0; k < kMaxSplit; ++k) {
                if (k < p.split_s) {
                  const float4 ok4 = k == piece ? make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                                              __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]))
                                                : pp[k][e];
                  if (k == 0) {
                    acc = make_float4(wk[0] * ok4.x, wk[0] * ok4.y, wk[0] * ok4.z, wk[0] * ok4.w);
                  } else {
                    acc = make_float4(fmaf(wk[k], ok4.x, acc.x), fmaf(wk[k], ok4.y, acc.y), fmaf(wk[k], ok4.z, acc.z),
                                      fmaf(wk[k], ok4.w, acc.w));
                  }
                }
              }
              o[4 * e] = __float_as_uint(acc.x);
              o[4 * e + 1] = __float_as_uint(acc.y);
              o[4 * e + 2] = __float_as_uint(acc.z);
              o[4 * e + 3] = __float_as_uint(acc.w);
            }
          }
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
  }

  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace zi
