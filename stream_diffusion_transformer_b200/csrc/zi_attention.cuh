// Non-causal flash attention (head_dim 128, bf16 in/out, fp32 softmax) on tcgen05.
//
// One CTA per (128-query tile, head, batch element), 6 warps:
//   warp 0      TMA: Q tile once, then K and V tiles (128 keys each) into
//               2-deep rings, straight out of the fused [rows, 3D] projection
//               buffer (the head's 128 columns as two 64-wide swizzled boxes)
//   warp 1      TMEM allocator + tcgen05.mma issuer:
//                 S_j = Q K_j^T          (A = Q smem, B = K smem, both K-major)
//                 O  += P_{j-1} V_{j-1}  (A = P smem K-major, B = V smem MN-major)
//               S is double-buffered in TMEM (2 x 128 columns), O lives in TMEM
//               (128 columns); S_{j+1} is issued before P_j V_j so the tensor
//               core keeps working while the softmax warps exponentiate.
//   warps 2..5  softmax: one thread per query row (its TMEM lane), online
//               softmax in the exp2 domain with a lazily updated running max
//               (O in TMEM is rescaled only when a row's max grows by more
//               than 2^8), P written to smem as bf16 in the swizzled layout
//               the MMA reads; final O / l written as bf16.
// The key sequence of a batch element can be split over two row segments of
// the token buffer (image rows and text rows); key tiles that run past a
// segment's end are masked to -inf.
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
  float scale_log2; // log2(e) / sqrt(head_dim)
};

namespace attn {
constexpr uint32_t kTile = 128 * 128 * 2;  // one 128 x 128 bf16 tile (two 64-column halves)
constexpr uint32_t kHalf = kTile / 2;
constexpr uint32_t kQ = 0, kK0 = kTile, kV0 = 3 * kTile, kP = 5 * kTile;
constexpr uint32_t kBar = 6 * kTile;
constexpr uint32_t kSmemBytes = kBar + 256 + 1024;
}  // namespace attn

ZI_DEV void attn_tile_rows(const AttnParams& p, int b, int tile, int& row0, int& valid) {
  int seg = 0;
  int t = tile;
  const int n0 = (p.seg_len[0] + 127) / 128;
  if (p.nseg > 1 && t >= n0) {
    seg = 1;
    t -= n0;
  }
  row0 = p.seg_row0[seg] + b * p.seg_len[seg] + t * 128;
  valid = min(128, p.seg_len[seg] - t * 128);
}

__global__ void __launch_bounds__(192, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm, AttnParams p) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2]
  uint64_t* s_free = bars + 11;  // [2]
  uint64_t* p_full = bars + 13;
  uint64_t* p_free = bars + 14;
  uint64_t* o_full = bars + 15;
  uint64_t* drain = bars + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (device_error_set()) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.y, b = blockIdx.z;
  int n_kv = (p.seg_len[0] + 127) / 128;
  if (p.nseg > 1) n_kv += (p.seg_len[1] + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(p_free, 1);
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tm);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int q_row0, q_valid;
  attn_tile_rows(p, b, blockIdx.x, q_row0, q_valid);
  const int colq = head * 128, colk = p.dim + head * 128, colv = 2 * p.dim + head * 128;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, kTile);
      tma_load_2d(smem + kQ, &tm, q_full, colq, q_row0);
      tma_load_2d(smem + kQ + kHalf, &tm, q_full, colq + 64, q_row0);
      uint32_t issued_k = 0, issued_v = 0;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        const int bi = j & 1;
        const uint32_t r = uint32_t(j) >> 1;
        int kv0, kvn;
        attn_tile_rows(p, b, j, kv0, kvn);
        if (!mbar_wait(&k_empty[bi], (r & 1u) ^ 1u, abort_flag, ZI_DEVERR_TIMEOUT_PRODUCER)) { ok = false; break; }
        mbar_arrive_expect_tx(&k_full[bi], kTile);
        tma_load_2d(smem + kK0 + bi * kTile, &tm, &k_full[bi], colk, kv0);
        tma_load_2d(smem + kK0 + bi * kTile + kHalf, &tm, &k_full[bi], colk + 64, kv0);
        ++issued_k;
        if (!mbar_wait(&v_empty[bi], (r & 1u) ^ 1u, abort_flag, ZI_DEVERR_TIMEOUT_PRODUCER)) { ok = false; break; }
        mbar_arrive_expect_tx(&v_full[bi], kTile);
        tma_load_2d(smem + kV0 + bi * kTile, &tm, &v_full[bi], colv, kv0);
        tma_load_2d(smem + kV0 + bi * kTile + kHalf, &tm, &v_full[bi], colv + 64, kv0);
        ++issued_v;
      }
      if (!ok) {
        volatile int never = 0;
        mbar_wait(q_full, 0, &never, ZI_DEVERR_TIMEOUT_DRAIN);
        for (uint32_t j = (issued_k > 2 ? issued_k - 2 : 0); j < issued_k; ++j)
          mbar_wait(&k_full[j & 1], (j >> 1) & 1u, &never, ZI_DEVERR_TIMEOUT_DRAIN);
        for (uint32_t j = (issued_v > 2 ? issued_v - 2 : 0); j < issued_v; ++j)
          mbar_wait(&v_full[j & 1], (j >> 1) & 1u, &never, ZI_DEVERR_TIMEOUT_DRAIN);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 128, false, true);
      const uint32_t q_addr = smem_u32(smem + kQ);
      const uint32_t p_addr = smem_u32(smem + kP);
      bool ok = mbar_wait(q_full, 0, abort_flag, ZI_DEVERR_TIMEOUT_MMA);
      tc_fence_after();
      auto issue_pv = [&](int jj) -> bool {
        const int bb = jj & 1;
        const uint32_t rr = uint32_t(jj) >> 1;
        if (!mbar_wait(p_full, uint32_t(jj) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA)) return false;
        if (!mbar_wait(&v_full[bb], rr & 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + kV0 + bb * kTile);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = smem_desc_sw128(p_addr + (k >> 2) * kHalf + (k & 3) * 32, 16);
          const uint64_t bd = smem_desc_sw128(v_addr + k * 2048, kHalf);
          tc_mma(tmem + 256, ad, bd, idesc_o, (jj > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(&v_empty[bb]);
        tc_commit(p_free);
        return true;
      };
      for (int j = 0; j < n_kv && ok; ++j) {
        const int bi = j & 1;
        const uint32_t r = uint32_t(j) >> 1;
        if (!mbar_wait(&k_full[bi], r & 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA)) { ok = false; break; }
        if (!mbar_wait(&s_free[bi], (r & 1u) ^ 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + kK0 + bi * kTile);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = smem_desc_sw128(q_addr + (k >> 2) * kHalf + (k & 3) * 32, 16);
          const uint64_t bd = smem_desc_sw128(k_addr + (k >> 2) * kHalf + (k & 3) * 32, 16);
          tc_mma(tmem + uint32_t(bi * 128), ad, bd, idesc_s, k > 0 ? 1u : 0u);
        }
        tc_commit(&k_empty[bi]);
        tc_commit(&s_full[bi]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && issue_pv(n_kv - 1)) {
        tc_commit(o_full);
      } else {
        tc_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, ZI_DEVERR_TIMEOUT_DRAIN);
      }
    }
  } else {
    const int q = warp & 3;
    const int i = q * 32 + lane;  // query row in the tile == TMEM lane
    const uint32_t lane_addr = tmem + (uint32_t(q * 32) << 16);
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l = 0.f;
    uint32_t s[128];
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int bi = j & 1;
      const uint32_t r = uint32_t(j) >> 1;
      int kv0, kvn;
      attn_tile_rows(p, b, j, kv0, kvn);
      if (!mbar_wait(&s_full[bi], r & 1u, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(lane_addr + uint32_t(bi * 128 + c * 32), &s[c * 32]);
      }
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence32(&s[c * 32]);
      tc_fence_before();
      mbar_arrive(&s_free[bi]);

      // Row max and row sum use 8 independent chains each, so the per-element
      // FMNMX / FFMA / EX2 / FADD of different columns overlap instead of
      // waiting on one serial dependency chain.
      if (kvn < 128) {  // the segment's last key tile: mask the columns past its end
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= kvn) s[c] = __float_as_uint(-INFINITY);
      }
      float mxs[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mxs[k] = __uint_as_float(s[k]);
#pragma unroll
      for (int c = 8; c < 128; ++c) mxs[c & 7] = fmaxf(mxs[c & 7], __uint_as_float(s[c]));
      const float mx = fmaxf(fmaxf(fmaxf(mxs[0], mxs[1]), fmaxf(mxs[2], mxs[3])),
                             fmaxf(fmaxf(mxs[4], mxs[5]), fmaxf(mxs[6], mxs[7])));
      const float m_new = fmaxf(m_run, mx * sl2);
      const bool need = m_new > m_run + 8.0f;
      float alpha = 1.0f;
      const bool resc = __any_sync(0xffffffffu, need);
      if (resc) {
        alpha = fast_exp2(m_run - m_new);
        m_run = m_new;
        l *= alpha;
      }
      const float neg_m = -m_run;
      float sums[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) sums[k] = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const float e = fast_exp2(fmaf(__uint_as_float(s[c]), sl2, neg_m));
        sums[c & 7] += e;
        s[c] = __float_as_uint(e);
      }
      l += ((sums[0] + sums[1]) + (sums[2] + sums[3])) + ((sums[4] + sums[5]) + (sums[6] + sums[7]));
      if (j >= 1) {
        if (!mbar_wait(p_free, uint32_t(j - 1) & 1u, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX)) { ok = false; break; }
        tc_fence_after();
        if (resc) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32_sync(lane_addr + 256 + c * 32, o);
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(lane_addr + 256 + c * 32, o);
          }
          tmem_wait_st();
        }
      }
      // P row i -> smem, two 64-column halves, 16-byte chunks swizzled by (i & 7)
      uint8_t* prow = smem + kP + i * 128;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const int c0 = h * 64 + c8 * 8;
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(s[c0 + 0]), __uint_as_float(s[c0 + 1]));
          w.y = pack_bf16x2(__uint_as_float(s[c0 + 2]), __uint_as_float(s[c0 + 3]));
          w.z = pack_bf16x2(__uint_as_float(s[c0 + 4]), __uint_as_float(s[c0 + 5]));
          w.w = pack_bf16x2(__uint_as_float(s[c0 + 6]), __uint_as_float(s[c0 + 7]));
          *reinterpret_cast<uint4*>(prow + h * kHalf + ((c8 ^ (i & 7)) << 4)) = w;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && mbar_wait(o_full, 0, abort_flag, ZI_DEVERR_TIMEOUT_SOFTMAX)) {
      tc_fence_after();
      const float inv = 1.0f / l;
      uint16_t* orow = p.out + size_t(q_row0 + i) * p.ldo + head * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32_sync(lane_addr + 256 + c * 32, o);
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

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace zi
