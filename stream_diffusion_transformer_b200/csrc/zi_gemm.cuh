// Persistent GEMM for sm_100a with fused epilogues:  C[M, N] = A[M, K] * B[N, K]^T,
// operands bf16 (kind::f16) or e4m3 with per-row scales (kind::f8f6f4).
//
// A is the activation (row-major, K contiguous); B is a weight in the
// checkpoint's own [out, in] orientation, which is exactly the K-major operand
// tcgen05 wants, so weights are used as stored.
//
// Two kernels share one structure, 10 warps per CTA:
//   warp 0      TMA producer: a 128-row A tile + a B tile of 128 bytes of K per
//               stage (64 bf16 or 128 e4m3), 128-byte swizzle, STAGES-deep ring
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//               (32 bytes of K per instruction; fp32 accumulator in TMEM)
//   warps 2..9  epilogue in two groups of four (each covers all 128 TMEM lanes and
//               one half of the tile's columns): tcgen05.ld TMEM -> registers ->
//               fused math -> global
// gemm_tn_body: one CTA per SM computes 128 x BN tiles (M = 128 MMAs, a BN-row B
// tile per stage).  gemm_pair_body: a cluster of two CTAs on two SMs computes
// 256 x 256 tiles with cta_group::2 MMAs (M = 256) issued by CTA 0; each CTA stages
// its own 128 rows of A and its 128-row half of B (see the comment above it).
// The accumulator is double-buffered in TMEM (2 x BN columns), so the epilogue
// of tile i overlaps the main loop of tile i + 1.  Tiles are walked in groups that
// keep one operand's panels in L2 while the other is swept (tile_origin).
#pragma once
#include "zi_common.cuh"

// Schedule functions callable from host code too (tests/schedule_check.cu runs them on the CPU).
#define ZI_HD __host__ __device__ __forceinline__

namespace zi {

// Maps a global row of the token buffer to its batch element and to its index
// in one sequence's position table.  Rows [0, n_a) hold segment A (len_a rows
// per batch element), rows [n_a, ...) hold segment B (len_b rows per element);
// in a sequence, segment A occupies positions [0, len_a) and B [len_a, len_a + len_b).
// tab_stride: rows of the position (RoPE) table per batch element; 0 when the
// elements share one table, len_a + len_b when each element has its own.
struct RowMap {
  int n_a, len_a, len_b;
  int tab_stride;
  ZI_DEV int batch(int r) const { return r < n_a ? r / len_a : (r - n_a) / len_b; }
  ZI_DEV int pos(int r) const { return r < n_a ? r % len_a : len_a + (r - n_a) % len_b; }
  ZI_DEV int tab(int r) const { return (tab_stride ? batch(r) * tab_stride : 0) + pos(r); }
};

enum EpiKind : int {
  EPI_BF16 = 0,     // out bf16 [M, ldo]
  EPI_F32_BIAS = 1, // out fp32 [M, ldo] = acc + bias
  EPI_QKV = 2,      // q, k: RMSNorm over each 128-wide head, gain, RoPE; v: plain; out bf16 [M, 3D]
  EPI_SWIGLU = 3,   // 256-wide tile = 128 gate + 128 up columns -> out bf16 SiLU(gate) * up [M, N/2]
  EPI_UNPATCH = 4,  // final linear: acc + bias scattered to the latent [B, C, H, W] fp32
};

struct EpiParams {
  void* out;
  int ldo;                 // row stride of `out` in elements
  const uint16_t* bias;    // bf16 [N] (EPI_F32_BIAS, EPI_UNPATCH)
  const float2* rope;      // (cos, sin) [head_dim / 2][rope_n]: pair-major, so a warp's 32 rows
  int rope_n;              // (consecutive positions) read one pair in one coalesced load (EPI_QKV)
  const uint16_t* g_q;     // bf16 [128] QK-RMSNorm gains (EPI_QKV)
  const uint16_t* g_k;
  float eps;
  int dim;                 // D: column offset of k in the fused projection (EPI_QKV)
  int row_off;             // global row of local row 0 (for RowMap)
  RowMap map;
  int s_img, grid_w, lat_c, lat_h, lat_w;  // EPI_UNPATCH
  const float* a_scale;  // e4m3 operands: per-row scale of A [M] ...
  const float* b_scale;  // ... and of B [N] (per output column)
};

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr uint32_t kABytes = 128u * 64u * 2u;
  static constexpr uint32_t kBBytes = uint32_t(BN) * 64u * 2u;
  static constexpr uint32_t kStage = kABytes + kBBytes;
  static constexpr uint32_t kBarOff = STAGES * kStage;
  static constexpr uint32_t kBytes = kBarOff + 256u + 1024u;  // + barriers/flags (< 256 B) + alignment slack
  static constexpr uint32_t kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                        : (2 * BN <= 256) ? 256 : 512;
};

// Store 32 fp32 values as bf16 (64 contiguous bytes).
ZI_DEV void store_bf16x32(uint16_t* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = w;
  }
}

// Epilogue of one half of a tile (`half` 0 or 1: two groups of 4 epilogue warps
// share each tile), for the tile starting at output column n0.  Generic epilogues
// take columns [half BN/2, (half + 1) BN/2); QKV one 128-wide head each; SwiGLU
// the gate/up pairs [64 half, 64 half + 64).
// acc[i] *= sa * b_scale[col + i] for 32 accumulator columns (e4m3 operands).
ZI_DEV void scale_acc32(uint32_t* v, float sa, const float* b_scale, int col) {
  const float4* bs = reinterpret_cast<const float4*>(b_scale + col);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 w = __ldg(bs + q);
    v[4 * q] = __float_as_uint(__uint_as_float(v[4 * q]) * (sa * w.x));
    v[4 * q + 1] = __float_as_uint(__uint_as_float(v[4 * q + 1]) * (sa * w.y));
    v[4 * q + 2] = __float_as_uint(__uint_as_float(v[4 * q + 2]) * (sa * w.z));
    v[4 * q + 3] = __float_as_uint(__uint_as_float(v[4 * q + 3]) * (sa * w.w));
  }
}

template <int EPI, int BN, bool F8>
ZI_DEV void gemm_epilogue(uint32_t tbase, int row, bool row_ok, int n0, int half, const EpiParams& ep) {
  constexpr int kChunks = BN / 64;  // 32-column chunks per half
  static_assert(!F8 || EPI == EPI_BF16 || EPI == EPI_QKV || EPI == EPI_SWIGLU, "e4m3 epilogues: bf16, QKV, SwiGLU");
  uint32_t v[32];
  float f[32];
  const float sa = (F8 && row_ok) ? __ldg(ep.a_scale + row) : 1.f;
  if constexpr (EPI == EPI_BF16 || EPI == EPI_F32_BIAS) {
#pragma unroll 1
    for (int c = half * kChunks; c < (half + 1) * kChunks; ++c) {
      tmem_ld32_sync(tbase + c * 32, v);
      if (row_ok) {
        const int col = n0 + c * 32;
        if constexpr (F8) scale_acc32(v, sa, ep.b_scale, col);
        if constexpr (EPI == EPI_BF16) {
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
          store_bf16x32(static_cast<uint16_t*>(ep.out) + size_t(row) * ep.ldo + col, f);
        } else {
          float4* d = reinterpret_cast<float4*>(static_cast<float*>(ep.out) + size_t(row) * ep.ldo + col);
          const uint4* bp = reinterpret_cast<const uint4*>(ep.bias + col);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 b = __ldg(bp + q);
            const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float4 o;
              o.x = __uint_as_float(v[8 * q + 4 * h + 0]) + bf16_to_f32(uint16_t(bw[2 * h] & 0xFFFF));
              o.y = __uint_as_float(v[8 * q + 4 * h + 1]) + bf16_to_f32(uint16_t(bw[2 * h] >> 16));
              o.z = __uint_as_float(v[8 * q + 4 * h + 2]) + bf16_to_f32(uint16_t(bw[2 * h + 1] & 0xFFFF));
              o.w = __uint_as_float(v[8 * q + 4 * h + 3]) + bf16_to_f32(uint16_t(bw[2 * h + 1] >> 16));
              d[2 * q + h] = o;
            }
          }
        }
      }
    }
  } else if constexpr (EPI == EPI_QKV) {
    static_assert(BN == 256, "QKV epilogue works on 128-wide heads (two per full tile)");
    const int region = n0 / ep.dim;  // 0 = q, 1 = k, 2 = v
    uint16_t* orow = static_cast<uint16_t*>(ep.out) + size_t(row) * ep.ldo;
    if (region == 2) {
#pragma unroll 1
      for (int c = half * kChunks; c < (half + 1) * kChunks; ++c) {
        tmem_ld32_sync(tbase + c * 32, v);
        if (row_ok) {
          if constexpr (F8) scale_acc32(v, sa, ep.b_scale, n0 + c * 32);
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
          store_bf16x32(orow + n0 + c * 32, f);
        }
      }
      return;
    }
    const uint16_t* g = region == 0 ? ep.g_q : ep.g_k;
    const int p = row_ok ? ep.map.tab(row + ep.row_off) : 0;
    const float2* rp = ep.rope + p;  // pair j at rp[j * rope_n]
#pragma unroll 1
    for (int hh = half; hh < half + 1; ++hh) {  // one 128-wide head per half
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        tmem_ld32_sync(tbase + hh * 128 + c * 32, v);
        if constexpr (F8) scale_acc32(v, sa, ep.b_scale, n0 + hh * 128 + c * 32);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x = __uint_as_float(v[i]);
          ss = fmaf(x, x, ss);
        }
      }
      const float r = rsqrtf(ss * (1.0f / 128.0f) + ep.eps);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        tmem_ld32_sync(tbase + hh * 128 + c * 32, v);
        if (row_ok) {
          if constexpr (F8) scale_acc32(v, sa, ep.b_scale, n0 + hh * 128 + c * 32);
          uint4 gw[4];  // the 32 gains of this chunk (the same for every row: broadcast loads)
#pragma unroll
          for (int k = 0; k < 4; ++k) gw[k] = __ldg(reinterpret_cast<const uint4*>(g + c * 32) + k);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t gp = (i & 3) == 0 ? gw[i >> 2].x : (i & 3) == 1 ? gw[i >> 2].y
                              : (i & 3) == 2 ? gw[i >> 2].z : gw[i >> 2].w;  // gains of dims 2i, 2i + 1
            const float a = __uint_as_float(v[2 * i]) * r * __uint_as_float(gp << 16);
            const float b = __uint_as_float(v[2 * i + 1]) * r * __uint_as_float(gp & 0xFFFF0000u);
            const float2 cs = __ldg(rp + size_t(c * 16 + i) * ep.rope_n);
            f[2 * i] = a * cs.x - b * cs.y;
            f[2 * i + 1] = a * cs.y + b * cs.x;
          }
          store_bf16x32(orow + n0 + hh * 128 + c * 32, f);
        }
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    static_assert(BN == 256, "SwiGLU epilogue pairs 128 gate with 128 up columns");
    uint32_t u[32];
    uint16_t* orow = static_cast<uint16_t*>(ep.out) + size_t(row) * ep.ldo + n0 / 2;
#pragma unroll 1
    for (int c = 2 * half; c < 2 * half + 2; ++c) {
      tmem_ld32(tbase + c * 32, v);
      tmem_ld32(tbase + 128 + c * 32, u);
      tmem_wait_ld();
      reg_fence32(v);
      reg_fence32(u);
      if (row_ok) {
        if constexpr (F8) {
          scale_acc32(v, sa, ep.b_scale, n0 + c * 32);
          scale_acc32(u, sa, ep.b_scale, n0 + 128 + c * 32);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float gt = __uint_as_float(v[i]);
          const float up = __uint_as_float(u[i]);
          f[i] = gt / (1.0f + __expf(-gt)) * up;
        }
        store_bf16x32(orow + c * 32, f);
      }
    }
  } else if constexpr (EPI == EPI_UNPATCH) {
    float* out = static_cast<float*>(ep.out);
    const int gr = row_ok ? row + ep.row_off : 0;
    const int b = gr / ep.s_img, t = gr % ep.s_img;
    const int ty = t / ep.grid_w, tx = t % ep.grid_w;
#pragma unroll 1
    for (int c = half * kChunks; c < (half + 1) * kChunks; ++c) {
      tmem_ld32_sync(tbase + c * 32, v);
      if (row_ok) {
#pragma unroll 4
        for (int i = 0; i < 32; ++i) {
          const int feat = n0 + c * 32 + i;
          const int ch = feat % ep.lat_c, pq = feat / ep.lat_c;
          const int y = 2 * ty + (pq >> 1), x = 2 * tx + (pq & 1);
          out[((size_t(b) * ep.lat_c + ch) * ep.lat_h + y) * ep.lat_w + x] =
              __uint_as_float(v[i]) + bf16_to_f32(__ldg(ep.bias + feat));
        }
      }
    }
  }
}

// Work schedule.  T output tiles of 128 x BN run on G persistent CTAs, tile t
// on CTA t % G.  When T % G leaves a last wave of R < G tiles, those R tiles are
// cut along K into s pieces (s R <= G, s <= kMaxSplit, at least kMinSplitKb
// k-blocks each), one piece per CTA, so the ragged wave costs about 1/s of a
// tile's time.  (Cutting along N instead would not help: a tcgen05.mma with
// A and B in shared memory takes about as long at N = 64 or 128 as at 256.)
// Every piece stores its fp32 partial tile in its own slot and bumps the tile's
// counter; the piece that completes the count adds the partials in slot order
// (the same order whichever piece finishes, so results are deterministic) and
// runs the fused epilogue.  No CTA waits for another.
constexpr int kMaxSplit = 4;
constexpr int kEpiWarps = 8;                        // two groups of 4 (each covers all 128 TMEM lanes)
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;   // + the TMA and MMA warps
constexpr int kMinSplitKb = 4;
constexpr int kSplitSlots = 160;  // partial slots (>= G); counters likewise

struct TailSched {
  int grid;        // G
  int dp_tiles;    // tiles [0, dp_tiles) run whole, walked with stride G
  int tail_s;      // K pieces per tail tile (1 = no tail)
  int tail_items;  // CTAs [0, tail_items) each run piece c % s of tile dp_tiles + c / s
  int kb;          // k-blocks per tile
  int num_n;       // N tiles
  int group;       // tiles per group along the grouped dimension (see tile_origin)
  int group_n;     // 1: groups of N tiles (B panels held in L2), 0: groups of M tiles
};

// Tile t covers rows [m0, m0 + BM) and columns [n0, n0 + BN).  Tiles are walked in
// groups: `group` M tiles (their A panels) swept over every N tile with M fastest
// inside the group, or `group` N tiles swept over every M tile with N fastest.  The
// CTAs running at the same time then read a few panels of the swept operand while
// the group's panels stay in L2 for the whole sweep, so from DRAM the grouped operand
// is read once and the swept one once per group (choose_raster picks the side and
// the group size from the operands' sizes).
template <int BM, int BN>
ZI_HD void tile_origin(const TailSched& s, int num_m, int tile, int& m0, int& n0) {
  if (s.group_n) {
    const int per = s.group * num_m;
    const int g = tile / per, r = tile - g * per;
    const int cols = s.group < s.num_n - g * s.group ? s.group : s.num_n - g * s.group;
    n0 = (g * s.group + r % cols) * BN;
    m0 = (r / cols) * BM;
  } else {
    const int per = s.group * s.num_n;
    const int g = tile / per, r = tile - g * per;
    const int rows = s.group < num_m - g * s.group ? s.group : num_m - g * s.group;
    m0 = (g * s.group + r % rows) * BM;
    n0 = (r / rows) * BN;
  }
}

// Bytes of one operand's panels a group may keep in L2 (about 45% of the 126 MB, so
// the swept operand's tiles, the output and other traffic still fit beside them).
constexpr double kRasterL2Budget = 56.0e6;

// Picks the grouped side and group size with the fewest DRAM bytes: grouping M tiles
// reads A once and B once per group, grouping N tiles the reverse.  a_panel / b_panel:
// bytes of one M tile's rows of A / one N tile's rows of B over the whole K.
inline void choose_raster(int num_m, int num_n, double a_panel, double b_panel, int& group, int& group_n) {
  auto fit = [](double panel, int n) {
    int g = panel > 0 ? int(kRasterL2Budget / panel) : n;
    return g < 1 ? 1 : (g > n ? n : g);
  };
  const int gm = fit(a_panel, num_m), gn = fit(b_panel, num_n);
  const double tm = num_m * a_panel + double((num_m + gm - 1) / gm) * num_n * b_panel;
  const double tn = num_n * b_panel + double((num_n + gn - 1) / gn) * num_m * a_panel;
  if (tn < tm) {
    group = gn;
    group_n = 1;
  } else {
    group = gm;
    group_n = 0;
  }
}

// Units (CTAs, or CTA pairs) a launch needs: one per tile up to G, or one per tail piece.
inline int sched_units(const TailSched& s, int tiles) {
  const int u = tiles < s.grid ? tiles : s.grid;
  return s.tail_items > u ? s.tail_items : u;
}

inline TailSched make_tail_sched(int tiles, int grid, int kb, bool can_split, int num_n, int group, int group_n) {
  TailSched s{grid, tiles, 1, 0, kb, num_n, group, group_n};
  const int rounds = tiles / grid, rest = tiles - rounds * grid;
  if (!can_split || rest == 0 || grid > kSplitSlots) return s;
  int f = grid / rest;
  if (f > kMaxSplit) f = kMaxSplit;
  if (f > kb / kMinSplitKb) f = kb / kMinSplitKb;
  if (f < 2) return s;
  s.dp_tiles = rounds * grid;
  s.tail_s = f;
  s.tail_items = f * rest;
  return s;
}

struct WorkItem {
  int tile;      // 128 x BN tile index (M fastest)
  int kb0, kb1;  // k-block range of this item
  int piece;     // -1: the whole tile; else the piece index of a split tail tile
};

// Walks one CTA's work items; every warp role walks the same sequence.
struct WorkWalker {
  const TailSched& s;
  int c, next_dp;
  bool tail_done;
  ZI_HD WorkWalker(const TailSched& sched, int cta) : s(sched), c(cta), next_dp(cta), tail_done(false) {}
  ZI_HD bool next(WorkItem& w) {
    if (next_dp < s.dp_tiles) {
      w.tile = next_dp;
      w.kb0 = 0;
      w.kb1 = s.kb;
      w.piece = -1;
      next_dp += s.grid;
      return true;
    }
    if (!tail_done && c < s.tail_items) {
      tail_done = true;
      w.tile = s.dp_tiles + c / s.tail_s;
      w.piece = c % s.tail_s;
      w.kb0 = w.piece * s.kb / s.tail_s;
      w.kb1 = (w.piece + 1) * s.kb / s.tail_s;
      return true;
    }
    return false;
  }
};

// Scratch of the split tail: partial tiles [kSplitSlots][BN / 4][128] float4
// (column-quad major, so a warp's 32 rows store 512 contiguous bytes) and one
// counter per tail tile, zero on entry (each tile's finisher puts it back to zero).
struct SplitScratch {
  float4* partials;
  int* counters;
};

// The persistent GEMM, for bf16 operands (F8 = false: kind::f16, 64 elements per
// 128-byte smem row) or e4m3 operands (F8 = true: kind::f8f6f4, 128 elements per
// row, accumulator scaled by ep.a_scale[row] * ep.b_scale[col] in the epilogue).
// The stage layout, swizzle and MMA count per stage (4) are the same for both.
template <int BN, int STAGES, int EPI, bool F8>
ZI_DEV void gemm_tn_body(const CUtensorMap& tmA, const CUtensorMap& tmB, int M, const EpiParams& ep,
                         const TailSched& sched, const SplitScratch& sk) {
  using L = GemmSmem<BN, STAGES>;
  constexpr int BM = 128, BK = F8 ? 128 : 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* ebar = drain + 1;  // the epilogue warps' own barrier (split tail)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ebar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;

  if (device_error_set()) return;  // an earlier kernel timed out: leave everything untouched
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    mbar_init(ebar, 32 * kEpiWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_m = (M + BM - 1) / BM;
  WorkItem wi;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      WorkWalker walk(sched, blockIdx.x);
      while (ok && walk.next(wi)) {
        int m0, n0;
        tile_origin<BM, BN>(sched, num_m, wi.tile, m0, n0);
        const uint32_t bytes = L::kStage;
        for (int kb = wi.kb0; kb < wi.kb1; ++kb) {
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&empty[s], (r & 1u) ^ 1u, abort_flag, ZI_DEVERR_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * L::kStage;
          mbar_arrive_expect_tx(&full[s], bytes);
          tma_load_2d(sa, &tmA, &full[s], kb * BK, m0);
          tma_load_2d(sa + L::kABytes, &tmB, &full[s], kb * BK, n0);
          ++it;
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        const uint32_t n = it < uint32_t(STAGES) ? it : uint32_t(STAGES);
        for (uint32_t j = 1; j <= n; ++j) {
          const uint32_t k = it - j;
          volatile int never = 0;
          mbar_wait(&full[k % STAGES], (k / STAGES) & 1u, &never, ZI_DEVERR_TIMEOUT_DRAIN);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t it = 0;
      int local = 0;
      bool ok = true;
      WorkWalker walk(sched, blockIdx.x);
      constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(128, BN) : idesc_bf16_f32(128, BN, false, false);
      while (ok && walk.next(wi)) {
        const int acc = local & 1;
        const uint32_t u = uint32_t(local) >> 1;
        ++local;
        if (!mbar_wait(&tempty[acc], (u & 1u) ^ 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + uint32_t(acc * BN);
        for (int kb = wi.kb0; kb < wi.kb1; ++kb) {
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&full[s], r & 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * L::kStage);
          const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 32 bytes of K per MMA: 16 bf16 or 32 e4m3 elements
            const uint64_t ad = smem_desc_sw128(a_addr + k * 32, 16), bd = smem_desc_sw128(b_addr + k * 32, 16);
            const uint32_t acc_in = (kb != wi.kb0 || k != 0) ? 1u : 0u;
            if constexpr (F8) {
              tc_mma_f8(d, ad, bd, idesc, acc_in);
            } else {
              tc_mma(d, ad, bd, idesc, acc_in);
            }
          }
          tc_commit(&empty[s]);
          ++it;
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      if (!ok) {
        // Wait until every MMA issued so far has finished before TMEM is freed.
        tc_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, ZI_DEVERR_TIMEOUT_DRAIN);
      }
    }
  } else {
    const int q = warp & 3;             // this warp's TMEM lane quarter
    const int half = (warp - 2) >> 2;   // which half of the tile's columns
    const int row_in_tile = q * 32 + lane;
    int local = 0;
    uint32_t ephase = 0;
    auto epi_sync = [&]() -> bool {  // the epilogue threads meet (bounded wait)
      mbar_arrive(ebar);
      const bool r = mbar_wait(ebar, ephase, abort_flag, ZI_DEVERR_TIMEOUT_EPILOGUE);
      ephase ^= 1u;
      return r;
    };
    WorkWalker walk(sched, blockIdx.x);
    while (walk.next(wi)) {
      const int acc = local & 1;
      const uint32_t u = uint32_t(local) >> 1;
      ++local;
      if (!mbar_wait(&tfull[acc], u & 1u, abort_flag, ZI_DEVERR_TIMEOUT_EPILOGUE)) break;
      tc_fence_after();
      int m0, n0;
      tile_origin<BM, BN>(sched, num_m, wi.tile, m0, n0);
      const int row = m0 + row_in_tile;
      const uint32_t tb = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN);
      bool finish = true;
      if (wi.piece >= 0) {
        // A piece of a split tile: publish the partial, then finish only if last.
        const int slot0 = blockIdx.x - wi.piece;  // slot of piece 0 of this tile
        float4* mine = sk.partials + size_t(blockIdx.x) * (32 * BN) + row_in_tile;
        for (int c = half * (BN / 64); c < (half + 1) * (BN / 64); ++c) {
          uint32_t v[32];
          tmem_ld32_sync(tb + c * 32, v);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            __stcg(mine + size_t(c * 8 + k) * 128,
                   make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                               __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3])));
        }
        __threadfence();
        if (!epi_sync()) break;
        if (threadIdx.x == 64) {
          const int t = wi.tile - sched.dp_tiles;
          const int old = atomicAdd(&sk.counters[t], 1);
          const bool last = old == sched.tail_s - 1;
          if (last) sk.counters[t] = 0;  // ready for the next launch
          *last_flag = last ? 1 : 0;
        }
        if (!epi_sync()) break;
        finish = *last_flag != 0;
        if (finish) {
          __threadfence();
          for (int c = half * (BN / 64); c < (half + 1) * (BN / 64); ++c) {
            // Sum the pieces in piece order 0, 1, ..., s - 1 whichever piece finishes;
            // each other piece's 8 loads are issued together.
            uint32_t v[32];
            tmem_ld32_sync(tb + c * 32, v);
            float4 tot[8];
            for (int j = 0; j < sched.tail_s; ++j) {
              float4 pj[8];
              if (j == wi.piece) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  pj[k] = make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                      __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
              } else {
                const float4* src = sk.partials + size_t(slot0 + j) * (32 * BN) + size_t(c * 8) * 128 + row_in_tile;
#pragma unroll
                for (int k = 0; k < 8; ++k) pj[k] = __ldcg(src + size_t(k) * 128);
              }
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                if (j == 0) {
                  tot[k] = pj[k];
                } else {
                  tot[k].x += pj[k].x;
                  tot[k].y += pj[k].y;
                  tot[k].z += pj[k].z;
                  tot[k].w += pj[k].w;
                }
              }
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              v[4 * k] = __float_as_uint(tot[k].x);
              v[4 * k + 1] = __float_as_uint(tot[k].y);
              v[4 * k + 2] = __float_as_uint(tot[k].z);
              v[4 * k + 3] = __float_as_uint(tot[k].w);
            }
            tmem_st32(tb + c * 32, v);
          }
          tmem_wait_st();
          // Each warp group merged its own half of the columns; the SwiGLU epilogue
          // reads columns of both halves, so all merges finish before any epilogue.
          tc_fence_before();
          if (!epi_sync()) break;
          tc_fence_after();
        }
      }
      if (finish) gemm_epilogue<EPI, BN, F8>(tb, row, row < M, n0, half, ep);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ------------------------------------------------------------------ CTA-pair GEMM
// The same product on CTA pairs (tcgen05 cta_group::2): a pair computes a 256 x 256
// output tile, each CTA loading its own 128 rows of A and its own half (128 rows) of
// the tile's B, so a CTA moves 32 KB of operands per 64-deep (bf16) k-block instead of
// the 48 KB a 128 x 256 tile on one SM needs; CTA 0 issues M = 256 MMAs for both SMs,
// each CTA's TMEM holds its 128 rows x 256 columns (double-buffered), and each CTA's
// epilogue writes its own rows with the same fused epilogues.  Work units are the
// pair's tiles, walked like the single-CTA kernel's (tile_origin with BM = 256); a
// ragged last wave is cut along K the same way, each CTA keeping its own partials
// and counter for its 128 rows.
template <int STAGES>
struct PairSmem {
  static constexpr uint32_t kABytes = 128u * 128u;  // 128 rows x 128 bytes of K
  static constexpr uint32_t kBBytes = 128u * 128u;  // this CTA's 128 rows of the 256-row B tile
  static constexpr uint32_t kStage = kABytes + kBBytes;
  static constexpr uint32_t kBarOff = STAGES * kStage;
  static constexpr uint32_t kBytes = kBarOff + 256u + 1024u;
};

template <int STAGES, int EPI, bool F8>
ZI_DEV void gemm_pair_body(const CUtensorMap& tmA, const CUtensorMap& tmB, int M, const EpiParams& ep,
                           const TailSched& sched, const SplitScratch& sk) {
  using L = PairSmem<STAGES>;
  constexpr int BN = 256, BM = 256, BK = F8 ? 128 : 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);  // CTA 0: both CTAs' stage s loaded
  uint64_t* empty = full + STAGES;     // each CTA: its stage s consumed by the pair's MMAs
  uint64_t* tfull = empty + STAGES;    // each CTA: accumulator complete
  uint64_t* tempty = tfull + 2;        // CTA 0: both CTAs' epilogues drained the accumulator
  uint64_t* drain = tempty + 2;
  uint64_t* ebar = drain + 1;          // this CTA's epilogue warps' own barrier (split tail)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ebar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int unit = blockIdx.x >> 1;  // the pair's index in the work schedule

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kEpiWarps);  // one arrival per epilogue warp of each CTA
    }
    mbar_init(drain, 1);
    mbar_init(ebar, 32 * kEpiWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated before any remote access
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // an earlier kernel timed out: every role skips its work, both CTAs still meet at the end
  const bool err = device_error_set();

  const int num_m = (M + BM - 1) / BM;
  WorkItem wi;

  if (err) {
  } else if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      WorkWalker walk(sched, unit);
      while (walk.next(wi)) {
        int m0, n0;
        tile_origin<BM, BN>(sched, num_m, wi.tile, m0, n0);
        bool ok = true;
        for (int kb = wi.kb0; kb < wi.kb1; ++kb) {
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&empty[s], (r & 1u) ^ 1u, abort_flag, ZI_DEVERR_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * L::kStage;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * L::kStage);
          tma_load_2d_pair(sa, &tmA, &full[s], kb * BK, m0 + 128 * int(rank));
          tma_load_2d_pair(sa + L::kABytes, &tmB, &full[s], kb * BK, n0 + 128 * int(rank));
          ++it;
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      uint32_t it = 0;
      int local = 0;
      bool ok = true;
      WorkWalker walk(sched, unit);
      constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(256, BN) : idesc_bf16_f32(256, BN, false, false);
      while (ok && walk.next(wi)) {
        const int acc = local & 1;
        const uint32_t u = uint32_t(local) >> 1;
        ++local;
        if (!mbar_wait(&tempty[acc], (u & 1u) ^ 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + uint32_t(acc * BN);
        for (int kb = wi.kb0; kb < wi.kb1; ++kb) {
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&full[s], r & 1u, abort_flag, ZI_DEVERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * L::kStage);
          const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 32 bytes of K per MMA
            const uint64_t ad = smem_desc_sw128(a_addr + k * 32, 16), bd = smem_desc_sw128(b_addr + k * 32, 16);
            const uint32_t acc_in = (kb != wi.kb0 || k != 0) ? 1u : 0u;
            if constexpr (F8) {
              tc_mma2_f8(d, ad, bd, idesc, acc_in);
            } else {
              tc_mma2(d, ad, bd, idesc, acc_in);
            }
          }
          tc_commit_pair(&empty[s]);
          ++it;
        }
        if (ok) tc_commit_pair(&tfull[acc]);
      }
      if (!ok) {
        tc_commit_pair_local(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, ZI_DEVERR_TIMEOUT_DRAIN);
      }
    }
  } else {
    const int q = warp & 3;             // this warp's TMEM lane quarter
    const int half = (warp - 2) >> 2;   // which half of the tile's columns
    const int row_in_tile = q * 32 + lane;
    int local = 0;
    uint32_t ephase = 0;
    auto epi_sync = [&]() -> bool {  // this CTA's epilogue threads meet (bounded wait)
      mbar_arrive(ebar);
      const bool r = mbar_wait(ebar, ephase, abort_flag, ZI_DEVERR_TIMEOUT_EPILOGUE);
      ephase ^= 1u;
      return r;
    };
    WorkWalker walk(sched, unit);
    while (walk.next(wi)) {
      const int acc = local & 1;
      const uint32_t u = uint32_t(local) >> 1;
      ++local;
      if (!mbar_wait(&tfull[acc], u & 1u, abort_flag, ZI_DEVERR_TIMEOUT_EPILOGUE)) break;
      tc_fence_after();
      int m0, n0;
      tile_origin<BM, BN>(sched, num_m, wi.tile, m0, n0);
      const int row = m0 + 128 * int(rank) + row_in_tile;
      const uint32_t tb = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN);
      bool finish = true;
      if (wi.piece >= 0) {
        // A piece of a split tile: publish this CTA's partial, finish only if last
        // among the pieces' CTAs of the same rank.
        const int slot0 = 2 * (unit - wi.piece) + int(rank);  // piece 0's slot for this rank; piece j at slot0 + 2 j
        float4* mine = sk.partials + size_t(blockIdx.x) * (32 * BN) + row_in_tile;
        for (int c = half * (BN / 64); c < (half + 1) * (BN / 64); ++c) {
          uint32_t v[32];
          tmem_ld32_sync(tb + c * 32, v);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            __stcg(mine + size_t(c * 8 + k) * 128,
                   make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                               __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3])));
        }
        __threadfence();
        if (!epi_sync()) break;
        if (threadIdx.x == 64) {
          const int t = 2 * (wi.tile - sched.dp_tiles) + int(rank);
          const int old = atomicAdd(&sk.counters[t], 1);
          const bool last = old == sched.tail_s - 1;
          if (last) sk.counters[t] = 0;  // ready for the next launch
          *last_flag = last ? 1 : 0;
        }
        if (!epi_sync()) break;
        finish = *last_flag != 0;
        if (finish) {
          __threadfence();
          for (int c = half * (BN / 64); c < (half + 1) * (BN / 64); ++c) {
            uint32_t v[32];
            tmem_ld32_sync(tb + c * 32, v);
            float4 tot[8];
            for (int j = 0; j < sched.tail_s; ++j) {
              float4 pj[8];
              if (j == wi.piece) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  pj[k] = make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                      __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
              } else {
                const float4* src =
                    sk.partials + size_t(slot0 + 2 * j) * (32 * BN) + size_t(c * 8) * 128 + row_in_tile;
#pragma unroll
                for (int k = 0; k < 8; ++k) pj[k] = __ldcg(src + size_t(k) * 128);
              }
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                if (j == 0) {
                  tot[k] = pj[k];
                } else {
                  tot[k].x += pj[k].x;
                  tot[k].y += pj[k].y;
                  tot[k].z += pj[k].z;
                  tot[k].w += pj[k].w;
                }
              }
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              v[4 * k] = __float_as_uint(tot[k].x);
              v[4 * k + 1] = __float_as_uint(tot[k].y);
              v[4 * k + 2] = __float_as_uint(tot[k].z);
              v[4 * k + 3] = __float_as_uint(tot[k].w);
            }
            tmem_st32(tb + c * 32, v);
          }
          tmem_wait_st();
          // Each warp group merged its own half of the columns; the SwiGLU epilogue
          // reads columns of both halves, so all merges finish before any epilogue.
          tc_fence_before();
          if (!epi_sync()) break;
          tc_fence_after();
        }
      }
      if (finish) gemm_epilogue<EPI, BN, F8>(tb, row, row < M, n0, half, ep);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_leader(&tempty[acc]);
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
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512) : "memory");
  }
}

template <int STAGES, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M,
                          EpiParams ep, TailSched sched, SplitScratch sk) {
  gemm_pair_body<STAGES, EPI, false>(tmA, tmB, M, ep, sched, sk);
}

template <int STAGES, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_e4m3_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M,
                          EpiParams ep, TailSched sched, SplitScratch sk) {
  gemm_pair_body<STAGES, EPI, true>(tmA, tmB, M, ep, sched, sk);
}

template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_tn_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M,
                        EpiParams ep, TailSched sched, SplitScratch sk) {
  gemm_tn_body<BN, STAGES, EPI, false>(tmA, tmB, M, ep, sched, sk);
}

template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_e4m3_tn_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M,
                        EpiParams ep, TailSched sched, SplitScratch sk) {
  gemm_tn_body<BN, STAGES, EPI, true>(tmA, tmB, M, ep, sched, sk);
}

}  // namespace zi
