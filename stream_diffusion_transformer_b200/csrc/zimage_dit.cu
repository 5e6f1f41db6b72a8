// Host side of the C ABI declared in include/zimage_dit.h: argument checks,
// workspace carving, TMA descriptors and the stream-ordered launch sequence of
// the block and the full forward.  Nothing here allocates device memory or
// synchronises a stream (except zi_device_status / zi_clear_device_status).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "zi_attention.cuh"
#include "zi_common.cuh"
#include "zi_gemm.cuh"
#include "zi_rows.cuh"
#include "zimage_dit.h"

using namespace zi;

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kMaxDevices = 64;

// ---------------------------------------------------------------- device info

struct DevInfo {
  bool checked = false;
  bool ok = false;
  int sms = 0;
  unsigned attr_mask = 0;  // which kernels had their smem attribute raised on this device
};
DevInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device(DevInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZI_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.checked) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ZI_ERR_CUDA;
    d.ok = (major == 10 && minor == 0);
    d.sms = sms;
    d.checked = true;
  }
  *out = &d;
  return d.ok ? ZI_OK : ZI_ERR_DEVICE;
}

// Raise the dynamic shared-memory limit of `fn` once per device.
template <typename F>
int ensure_smem(DevInfo* d, unsigned bit, F fn, int bytes) {
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (d->attr_mask & (1u << bit)) return ZI_OK;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return ZI_ERR_CUDA;
  d->attr_mask |= 1u << bit;
  return ZI_OK;
}

// ---------------------------------------------------------------- TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

int encode_fn(EncodeTiledFn* out) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  *out = g_encode;
  return g_encode ? ZI_OK : ZI_ERR_CUDA;
}

// 2-D bf16 map over a row-major [outer, inner] matrix with rows `row_bytes`
// apart; box = box_inner x box_outer elements, 128-byte swizzle, zero fill.
int make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
             uint32_t box_inner, uint32_t box_outer,
             CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn enc;
  if (encode_fn(&enc) != ZI_OK) return ZI_ERR_CUDA;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) || (row_bytes & 15u)) return ZI_ERR_ALIGN;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ZI_OK : ZI_ERR_CUDA;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- launch profiling
// While enabled (zi_profile_begin .. zi_profile_end, per host thread) an event
// is recorded on the launching stream before the first kernel and after every
// kernel, so consecutive events bracket each launch.
struct Prof {
  bool on = false, started = false, overflow = false;
  int cap = 0, n = 0;
  std::vector<cudaEvent_t> ev;
  std::vector<int> kind;
};
thread_local Prof g_prof;

inline void prof_pre(cudaStream_t st) {
  if (g_prof.on && !g_prof.started) {
    cudaEventRecord(g_prof.ev[0], st);
    g_prof.started = true;
  }
}

// Status of the launch just made (+ the profiling marker after it).
inline int launched(int kind, cudaStream_t st) {
  if (cudaGetLastError() != cudaSuccess) return ZI_ERR_CUDA;
  if (g_prof.on) {
    if (g_prof.n < g_prof.cap) {
      cudaEventRecord(g_prof.ev[g_prof.n + 1], st);
      g_prof.kind[g_prof.n++] = kind;
    } else {
      g_prof.overflow = true;
    }
  }
  return ZI_OK;
}

#define ZI_TRY(expr)          \
  do {                        \
    const int _s = (expr);    \
    if (_s != ZI_OK) return _s; \
  } while (0)

// ---------------------------------------------------------------- GEMM

enum KernelBit : unsigned {
  BIT_GEMM_BF16 = 0,
  BIT_GEMM_F32 = 1,
  BIT_GEMM_QKV = 2,
  BIT_GEMM_SWIGLU = 3,
  BIT_GEMM_UNPATCH = 4,
  BIT_ATTN = 5,
  BIT_TMLP = 6,
};

constexpr int kStages = 4;

template <int BN, int EPI, bool F8>
struct GemmKernel {
  static constexpr auto fn = gemm_bf16_tn_kernel<BN, kStages, EPI>;
};
template <int BN, int EPI>
struct GemmKernel<BN, EPI, true> {
  static constexpr auto fn = gemm_e4m3_tn_kernel<BN, kStages, EPI>;
};

// A [M, K] and B [N, K] are bf16, or e4m3 codes with F8 (then ep.a_scale [M] and
// ep.b_scale [N] hold their per-row scales).  sk.partials == nullptr: no split
// tail (a caller without workspace).
template <int BN, int EPI, bool F8 = false>
int run_gemm(DevInfo* dev, unsigned bit, int kind, const void* A, const void* B, int M, int N, int K,
             const EpiParams& ep, cudaStream_t st, SplitScratch sk = SplitScratch{nullptr, nullptr}) {
  using L = GemmSmem<BN, kStages>;
  static_assert(BN <= 256, "split partial slots hold 128 x 256 fp32");
  constexpr int BK = F8 ? 128 : 64;  // elements per 128-byte smem row
  constexpr uint64_t esz = F8 ? 1 : 2;
  constexpr CUtensorMapDataType dt = F8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (M <= 0) return ZI_OK;
  if (K % BK != 0 || N % BN != 0 || K <= 0 || N <= 0) return ZI_ERR_SHAPE;
  if (F8 && (!ep.a_scale || !ep.b_scale)) return ZI_ERR_ARG;
  CUtensorMap ta, tb;
  ZI_TRY(make_map(&ta, A, uint64_t(K), uint64_t(M), uint64_t(K) * esz, BK, 128, dt));
  ZI_TRY(make_map(&tb, B, uint64_t(K), uint64_t(N), uint64_t(K) * esz, BK, BN, dt));
  auto kern = GemmKernel<BN, EPI, F8>::fn;
  ZI_TRY(ensure_smem(dev, bit + (F8 ? 8u : 0u), kern, int(L::kBytes)));
  const int tiles = ((M + 127) / 128) * (N / BN);
  int group, group_n;
  choose_raster((M + 127) / 128, N / BN, 128.0 * K * esz, double(BN) * K * esz, group, group_n);
  const TailSched sched =
      make_tail_sched(tiles, dev->sms, K / BK, sk.partials != nullptr, N / BN, group, group_n);
  const int grid = sched_units(sched, tiles);
  prof_pre(st);
  kern<<<grid, kGemmThreads, L::kBytes, st>>>(ta, tb, M, ep, sched, sk);
  return launched(kind, st);
}

// The same product on CTA pairs (256 x 256 tiles, B split across the pair; zi_gemm.cuh).
constexpr int kPairStages = 6;

template <int EPI, bool F8>
struct PairKernel {
  static constexpr auto fn = gemm_bf16_pair_kernel<kPairStages, EPI>;
};
template <int EPI>
struct PairKernel<EPI, true> {
  static constexpr auto fn = gemm_e4m3_pair_kernel<kPairStages, EPI>;
};

template <int EPI, bool F8 = false>
int run_gemm_pair(DevInfo* dev, unsigned bit, int kind, const void* A, const void* B, int M, int N, int K,
                  const EpiParams& ep, cudaStream_t st, SplitScratch sk = SplitScratch{nullptr, nullptr}) {
  using L = PairSmem<kPairStages>;
  constexpr int BK = F8 ? 128 : 64;
  constexpr uint64_t esz = F8 ? 1 : 2;
  constexpr CUtensorMapDataType dt = F8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (M <= 0) return ZI_OK;
  if (K % BK != 0 || N % 256 != 0 || K <= 0 || N <= 0) return ZI_ERR_SHAPE;
  if (F8 && (!ep.a_scale || !ep.b_scale)) return ZI_ERR_ARG;
  if (dev->sms < 2) return ZI_ERR_DEVICE;
  CUtensorMap ta, tb;
  ZI_TRY(make_map(&ta, A, uint64_t(K), uint64_t(M), uint64_t(K) * esz, BK, 128, dt));
  ZI_TRY(make_map(&tb, B, uint64_t(K), uint64_t(N), uint64_t(K) * esz, BK, 128, dt));
  auto kern = PairKernel<EPI, F8>::fn;
  ZI_TRY(ensure_smem(dev, bit + (F8 ? 24u : 16u), kern, int(L::kBytes)));
  const int pairs = dev->sms / 2;
  const int tiles = ((M + 255) / 256) * (N / 256);
  int group, group_n;
  choose_raster((M + 255) / 256, N / 256, 256.0 * K * esz, 256.0 * K * esz, group, group_n);
  const TailSched sched = make_tail_sched(tiles, pairs, K / BK, sk.partials != nullptr, N / 256, group, group_n);
  const int units = sched_units(sched, tiles);
  prof_pre(st);
  kern<<<2 * units, kGemmThreads, L::kBytes, st>>>(ta, tb, M, ep, sched, sk);
  return launched(kind, st);
}

// Which GEMMs of a block run on CTA pairs: those with at least this many rows.  On
// the B200 the pair kernel ran every projection of a 4,128-token block faster
// (QKV 6%, output 8%, FFN up 3%, FFN down 11%, same bits); below a few hundred rows
// the single-CTA kernel's 128-row tiles leave less of the last tile row idle.
constexpr int kPairMinRows = 512;

// The block's projections: CTA pairs when the shape favours them, else one CTA per tile.
template <int EPI, bool F8 = false>
int run_block_gemm(DevInfo* dev, unsigned bit, int kind, const void* A, const void* B, int M, int N, int K,
                   const EpiParams& ep, cudaStream_t st, SplitScratch sk) {
  if (M >= kPairMinRows) return run_gemm_pair<EPI, F8>(dev, bit, kind, A, B, M, N, K, ep, st, sk);
  return run_gemm<256, EPI, F8>(dev, bit, kind, A, B, M, N, K, ep, st, sk);
}

// bytes of one split-tail slot: a GEMM tile partial (128 x 256 fp32) or an attention
// piece (O of two query tiles plus their row max and sum), whichever is larger
constexpr size_t kSplitSlotBytes = size_t(128) * 256 * 4 > size_t(attn::kSlotF4) * 16 ? size_t(128) * 256 * 4
                                                                                       : size_t(attn::kSlotF4) * 16;

// Zeroes the split-tail counters of a workspace (once per forward; every tile's
// finisher puts its counter back to zero).
int clear_split(const SplitScratch& sk, cudaStream_t st) {
  prof_pre(st);
  zero_ints_kernel<<<1, 256, 0, st>>>(sk.counters, kSplitSlots);
  return launched(ZI_KERNEL_SPLIT_CLEAR, st);
}

EpiParams epi_plain(void* out, int ldo) {
  EpiParams e;
  memset(&e, 0, sizeof(e));
  e.out = out;
  e.ldo = ldo;
  e.map = RowMap{1, 1, 1, 0};
  return e;
}

// ---------------------------------------------------------------- attention

// sk.partials == nullptr: no split of the ragged last wave.
int run_attention(DevInfo* dev, const uint16_t* qkv, int qkv_rows, uint16_t* out, int dim, int heads, int batch,
                  int nseg, const int* row0, const int* len, const int* kv_len, cudaStream_t st,
                  SplitScratch sk = SplitScratch{nullptr, nullptr}) {
  CUtensorMap tm;
  ZI_TRY(make_map(&tm, qkv, uint64_t(3 * dim), uint64_t(qkv_rows), uint64_t(3 * dim) * 2, 64, 128));
  ZI_TRY(ensure_smem(dev, BIT_ATTN, attention_kernel, int(attn::kSmemBytes)));
  AttnParams p;
  memset(&p, 0, sizeof(p));
  p.out = out;
  p.ldo = dim;
  p.dim = dim;
  p.nseg = nseg;
  int qt = 0;
  for (int i = 0; i < 2; ++i) {
    p.seg_row0[i] = i < nseg ? row0[i] : 0;
    p.seg_len[i] = i < nseg ? len[i] : 1;
    if (i < nseg) qt += (len[i] + 127) / 128;
  }
  p.scale_log2 = float(1.4426950408889634 / std::sqrt(128.0));
  p.q_tiles = qt;
  p.kv_len = kv_len;
  p.pairs = (qt + 1) / 2;  // two query tiles per unit
  p.heads = heads;
  const long long units = static_cast<long long>(p.pairs) * heads * batch;
  if (units > 0x7fffffffLL / attn::kMaxSplit) return ZI_ERR_SHAPE;
  p.full_units = int(units);
  p.split_s = 1;
  const int G = dev->sms;
  const int rest = int(units % G);
  // fewest key tiles any element can have (each piece needs one)
  const int min_kv = (nseg > 1 ? (len[0] + 127) / 128 : 0) + (kv_len ? 1 : (len[nseg - 1] + 127) / 128);
  if (sk.partials && rest > 0 && G <= kSplitSlots) {
    int f = G / rest;
    if (f > attn::kMaxSplit) f = attn::kMaxSplit;
    if (f > min_kv) f = min_kv;
    if (f >= 2) {
      p.full_units = int(units) - rest;
      p.split_s = f;
      p.part = sk.partials;
      p.counters = sk.counters;
    }
  }
  const int grid = p.full_units + (int(units) - p.full_units) * p.split_s;
  prof_pre(st);
  attention_kernel<<<grid, attn::kThreads, attn::kSmemBytes, st>>>(tm, p);
  return launched(ZI_KERNEL_ATTENTION, st);
}

// ---------------------------------------------------------------- row kernels

// hq non-null: the output is e4m3 codes [rows][D] with per-row scales hs instead of bf16 h.
template <typename TIn>
int run_rms_mod(const TIn* x, int rows, int D, const uint16_t* gain, const float* scale, int scale_ld, RowMap map,
                int row_off, float eps, uint16_t* h, cudaStream_t st, uint8_t* hq = nullptr, float* hs = nullptr) {
  if (rows <= 0) return ZI_OK;
  prof_pre(st);
  rms_mod_kernel<TIn><<<rows, kRowThreads, 0, st>>>(x, D, gain, scale, scale_ld, map, row_off, eps, h, hq, hs);
  return launched(ZI_KERNEL_PRE_NORM, st);
}

// Per-row e4m3 codes and scales of a [rows, cols] fp32 or bf16 matrix (cols <= 16384).
constexpr int kQuantMaxCols = kRowThreads * 16 * 4;
template <typename TIn>
int run_quantize(const TIn* x, int rows, int cols, uint8_t* q, float* sc, cudaStream_t st) {
  if (rows <= 0) return ZI_OK;
  prof_pre(st);
  if (cols <= kRowThreads * kRowMaxVec * 4)
    quantize_rows_e4m3_kernel<TIn, kRowMaxVec><<<rows, kRowThreads, 0, st>>>(x, cols, q, sc);
  else
    quantize_rows_e4m3_kernel<TIn, 16><<<rows, kRowThreads, 0, st>>>(x, cols, q, sc);
  return launched(ZI_KERNEL_QUANTIZE, st);
}

int run_post(const PostParams& p, int rows, cudaStream_t st) {
  if (rows <= 0) return ZI_OK;
  prof_pre(st);
  post_residual_kernel<<<rows, kRowThreads, 0, st>>>(p);
  return launched(ZI_KERNEL_POST_NORM, st);
}

// ---------------------------------------------------------------- workspace

constexpr size_t kAlign = 1024;
inline size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct Ws {
  size_t mod, c, silu, hid, lens, pos, rope, x, h, hs, qkv, att, o, u, q8, q8s, tok, capn, split_cnt, split_part,
      total;
};

Ws carve(const zi_config& cfg, int batch, int s_img, int s_txt, bool model, int mod_cols) {
  const size_t D = size_t(cfg.dim);
  const size_t S = size_t(s_img) + size_t(s_txt);
  const size_t rows = size_t(batch) * S;
  const size_t Fp = size_t(zi_ffn_padded(cfg.ffn));
  const size_t pairs = size_t(cfg.head_dim) / 2;
  Ws w;
  size_t o = 0;
  w.mod = o; o = up(o + size_t(batch) * size_t(mod_cols) * 4);
  w.c = o; o = up(o + (model ? size_t(batch) * 256 * 4 : 0));
  w.silu = o; o = up(o + (model ? size_t(batch) * 256 * 4 : 0));
  w.hid = o; o = up(o + (model ? size_t(batch) * size_t(cfg.t_mid) * 4 : 0));
  // a model forward may give every batch element its own positions (text lengths)
  const size_t tab_rows = model ? rows : S;
  w.lens = o; o = up(o + (model ? size_t(batch) * 4 : 0));
  w.pos = o; o = up(o + (model ? tab_rows * 3 * 4 : 0));
  w.rope = o; o = up(o + tab_rows * pairs * 8);
  w.x = o; o = up(o + (model ? rows * D * 4 : 0));
  w.h = o; o = up(o + rows * D * 2);  // bf16 h, or e4m3 codes (rows x D bytes) for e4m3 blocks
  w.hs = o; o = up(o + rows * 4);      // per-row scales of e4m3 h
  w.qkv = o; o = up(o + rows * 3 * D * 2);
  w.att = o; o = up(o + rows * D * 2);
  w.o = o; o = up(o + rows * D * 2);
  w.u = o; o = up(o + rows * Fp * 2);
  // e4m3 codes of the attention output or of u (never live together) and their row scales
  w.q8 = o; o = up(o + rows * (Fp > D ? Fp : D));
  w.q8s = o; o = up(o + rows * 4);
  w.tok = o; o = up(o + (model ? size_t(batch) * s_img * size_t(4 * cfg.in_ch) * 2 : 0));
  w.capn = o; o = up(o + (model ? size_t(batch) * s_txt * size_t(cfg.cap_dim) * 2 : 0));
  w.split_cnt = o; o = up(o + size_t(kSplitSlots) * 4);
  w.split_part = o; o = up(o + size_t(kSplitSlots) * kSplitSlotBytes);
  w.total = o;
  return w;
}

int check_cfg(const zi_config* c) {
  if (!c) return ZI_ERR_ARG;
  if (c->head_dim != 128 || c->patch != 2) return ZI_ERR_SHAPE;
  if (c->dim <= 0 || c->dim % 256 != 0 || c->dim != c->heads * c->head_dim || c->dim > 4096) return ZI_ERR_SHAPE;
  if (c->rope_axes[0] + c->rope_axes[1] + c->rope_axes[2] != c->head_dim) return ZI_ERR_SHAPE;
  for (int i = 0; i < 3; ++i)
    if (c->rope_axes[i] <= 0 || c->rope_axes[i] % 2) return ZI_ERR_SHAPE;
  if (c->ffn <= 0 || c->cap_dim <= 0 || c->cap_dim % 64 != 0 || c->cap_dim > 4096) return ZI_ERR_SHAPE;
  if (c->t_freq != 256 || c->t_mid <= 0 || c->t_mid % 8) return ZI_ERR_SHAPE;  // warp-per-row timestep MLP
  if ((c->dim < 256 ? c->dim : 256) != 256) return ZI_ERR_SHAPE;  // adaLN GEMV is 256 wide
  if (4 * c->in_ch != 64) return ZI_ERR_SHAPE;                     // final linear uses a 64-wide tile
  if (c->n_noise < 0 || c->n_ctx < 0 || c->n_main < 1 || c->n_noise + c->n_main + 1 > kMaxAdaSegs)
    return ZI_ERR_SHAPE;
  return ZI_OK;
}

bool block_ptrs_ok(const zi_block_weights* w, bool need_mod) {
  if (!w) return false;
  const void* ps[] = {w->w_qkv, w->w_out, w->w13, w->w2, w->g_attn1, w->g_attn2, w->g_ffn1, w->g_ffn2, w->g_q, w->g_k};
  for (const void* p : ps)
    if (!p) return false;
  if (need_mod && (!w->w_ada || !w->b_ada)) return false;
  if ((w->w_ada == nullptr) != (w->b_ada == nullptr)) return false;
  // e4m3 projections: all four of w_qkv8, s_qkv, w13_8, s_13, or none; then optionally
  // all four of w_out8, s_out, w2_8, s_2
  const int nf8 = (w->w_qkv8 != nullptr) + (w->s_qkv != nullptr) + (w->w13_8 != nullptr) + (w->s_13 != nullptr);
  if (nf8 != 0 && nf8 != 4) return false;
  const int nf8b = (w->w_out8 != nullptr) + (w->s_out != nullptr) + (w->w2_8 != nullptr) + (w->s_2 != nullptr);
  if (nf8b != 0 && (nf8b != 4 || nf8 != 4)) return false;
  return true;
}

bool block_align_ok(const zi_block_weights* w) {
  const void* ps[] = {w->w_qkv, w->w_out, w->w13, w->w2, w->g_attn1, w->g_attn2, w->g_ffn1, w->g_ffn2, w->g_q, w->g_k};
  for (const void* p : ps)
    if (!aligned16(p)) return false;
  if (w->w_ada && !aligned16(w->w_ada)) return false;
  if (w->w_qkv8 && (!aligned16(w->w_qkv8) || !aligned16(w->s_qkv) || !aligned16(w->w13_8) || !aligned16(w->s_13)))
    return false;
  if (w->w_out8 && (!aligned16(w->w_out8) || !aligned16(w->s_out) || !aligned16(w->w2_8) || !aligned16(w->s_2)))
    return false;
  return true;
}

// How the gated residual after the FFN hands over to the next norm.
struct NextNormSpec {
  int kind;            // NEXT_NONE / NEXT_RMS / NEXT_LAYERNORM
  const uint16_t* gain;
  const float* scale;  // [B][mod_ld] or null
  int next_rows;       // h written for local rows < next_rows
  bool f8 = false;     // the next block takes e4m3 h (NEXT_RMS only)
};

// A block runs its QKV and FFN w1|w3 projections in e4m3 when it carries e4m3 weights
// for them, and also its output projection and FFN w2 when it carries those too.
inline bool block_f8(const zi_block_weights* w) { return w && w->w_qkv8 != nullptr; }
inline bool block_f8_all(const zi_block_weights* w) { return block_f8(w) && w->w_out8 != nullptr; }

// One block over `rows` rows of the token buffer starting at global row `row_off`.
// Pointers are local (row 0 = global row row_off).  h must already hold the
// block's pre-attention norm output.
struct BlockCtx {
  DevInfo* dev;
  const zi_config* cfg;
  const zi_block_weights* w;
  int rows, row_off, batch;
  RowMap map;
  float* x_in;
  float* x_out;
  uint16_t *h, *qkv, *att, *o, *u;
  uint8_t* hq;  // the same buffer as h, as e4m3 codes (D bytes per row) for e4m3 blocks
  float* hs;    // per-row scales of hq
  uint8_t* q8;  // e4m3 codes of att or u (all-e4m3 blocks), and ...
  float* q8s;   // ... their per-row scales
  const float2* rope;  // pair-major [head_dim / 2][rope_n]
  int rope_n;
  const float* mod;  // this block's 4D modulation inside the per-batch vector, or null
  int mod_ld;
  int nseg;
  int seg_row0[2], seg_len[2];  // local rows
  const int* kv_len;  // [batch] keys of the last segment (valid text tokens), or null = all
  SplitScratch split;  // split-tail scratch of the workspace (counters cleared)
};

int run_block(const BlockCtx& b, const NextNormSpec& next, cudaStream_t st) {
  const int D = b.cfg->dim;
  const int Fp = zi_ffn_padded(b.cfg->ffn);
  const float eps = b.cfg->norm_eps;
  // QKV projection with QK-RMSNorm + RoPE epilogue
  EpiParams eq = epi_plain(b.qkv, 3 * D);
  eq.rope = b.rope;
  eq.rope_n = b.rope_n;
  eq.g_q = b.w->g_q;
  eq.g_k = b.w->g_k;
  eq.eps = eps;
  eq.dim = D;
  eq.row_off = b.row_off;
  eq.map = b.map;
  const bool f8 = block_f8(b.w);
  if (f8) {
    eq.a_scale = b.hs;
    eq.b_scale = b.w->s_qkv;
    ZI_TRY((run_block_gemm<EPI_QKV, true>(b.dev, BIT_GEMM_QKV, ZI_KERNEL_GEMM_QKV, b.hq, b.w->w_qkv8, b.rows, 3 * D,
                                          D, eq, st, b.split)));
  } else {
    ZI_TRY((run_block_gemm<EPI_QKV>(b.dev, BIT_GEMM_QKV, ZI_KERNEL_GEMM_QKV, b.h, b.w->w_qkv, b.rows, 3 * D, D, eq,
                                    st, b.split)));
  }
  ZI_TRY(run_attention(b.dev, b.qkv, b.rows, b.att, D, b.cfg->heads, b.batch, b.nseg, b.seg_row0, b.seg_len,
                       b.kv_len, st, b.split));
  const bool f8all = block_f8_all(b.w);
  if (f8all) {
    ZI_TRY(run_quantize(b.att, b.rows, D, b.q8, b.q8s, st));
    EpiParams eo = epi_plain(b.o, D);
    eo.a_scale = b.q8s;
    eo.b_scale = b.w->s_out;
    ZI_TRY((run_block_gemm<EPI_BF16, true>(b.dev, BIT_GEMM_BF16, ZI_KERNEL_GEMM_OUT, b.q8, b.w->w_out8, b.rows, D,
                                           D, eo, st, b.split)));
  } else {
    ZI_TRY((run_block_gemm<EPI_BF16>(b.dev, BIT_GEMM_BF16, ZI_KERNEL_GEMM_OUT, b.att, b.w->w_out, b.rows, D, D,
                                     epi_plain(b.o, D), st, b.split)));
  }
  PostParams pa;
  memset(&pa, 0, sizeof(pa));
  pa.x_in = b.x_in;
  pa.x_out = b.x_out;
  pa.o = b.o;
  pa.g_post = b.w->g_attn2;
  pa.gate = b.mod ? b.mod + D : nullptr;
  pa.gate_ld = b.mod_ld;
  pa.next = NEXT_RMS;
  pa.g_next = b.w->g_ffn1;
  pa.scale = b.mod ? b.mod + 2 * D : nullptr;
  pa.scale_ld = b.mod_ld;
  pa.next_rows = b.rows;
  pa.h = b.h;
  pa.hq = f8 ? b.hq : nullptr;
  pa.hs = f8 ? b.hs : nullptr;
  pa.map = b.map;
  pa.row_off = b.row_off;
  pa.D = D;
  pa.eps = eps;
  pa.eps_ln = b.cfg->final_eps;
  ZI_TRY(run_post(pa, b.rows, st));
  if (f8) {
    EpiParams e13 = epi_plain(b.u, Fp);
    e13.a_scale = b.hs;
    e13.b_scale = b.w->s_13;
    ZI_TRY((run_block_gemm<EPI_SWIGLU, true>(b.dev, BIT_GEMM_SWIGLU, ZI_KERNEL_GEMM_FFN_UP, b.hq, b.w->w13_8, b.rows,
                                             2 * Fp, D, e13, st, b.split)));
  } else {
    ZI_TRY((run_block_gemm<EPI_SWIGLU>(b.dev, BIT_GEMM_SWIGLU, ZI_KERNEL_GEMM_FFN_UP, b.h, b.w->w13, b.rows, 2 * Fp,
                                       D, epi_plain(b.u, Fp), st, b.split)));
  }
  if (f8all) {
    ZI_TRY(run_quantize(b.u, b.rows, Fp, b.q8, b.q8s, st));
    EpiParams ed = epi_plain(b.o, D);
    ed.a_scale = b.q8s;
    ed.b_scale = b.w->s_2;
    ZI_TRY((run_block_gemm<EPI_BF16, true>(b.dev, BIT_GEMM_BF16, ZI_KERNEL_GEMM_FFN_DOWN, b.q8, b.w->w2_8, b.rows,
                                           D, Fp, ed, st, b.split)));
  } else {
    ZI_TRY((run_block_gemm<EPI_BF16>(b.dev, BIT_GEMM_BF16, ZI_KERNEL_GEMM_FFN_DOWN, b.u, b.w->w2, b.rows, D, Fp,
                                     epi_plain(b.o, D), st, b.split)));
  }
  PostParams pf = pa;
  pf.x_in = b.x_out;
  pf.g_post = b.w->g_ffn2;
  pf.gate = b.mod ? b.mod + 3 * D : nullptr;
  pf.next = next.kind;
  pf.g_next = next.gain;
  pf.scale = next.scale;
  pf.next_rows = next.next_rows;
  pf.hq = (next.kind == NEXT_RMS && next.f8) ? b.hq : nullptr;
  pf.hs = (next.kind == NEXT_RMS && next.f8) ? b.hs : nullptr;
  return run_post(pf, b.rows, st);
}

int run_ada(const AdaSegs& segs, const float* c, const float* silu_c, int batch, int out_ld, float* out,
            cudaStream_t st) {
  int max_rows = 0;
  for (int i = 0; i < segs.n; ++i) max_rows = segs.rows[i] > max_rows ? segs.rows[i] : max_rows;
  dim3 grid((max_rows + 63) / 64, segs.n);
  prof_pre(st);
  ada_gemv_kernel<<<grid, 256, 0, st>>>(segs, c, silu_c, batch, out_ld, out);
  return launched(ZI_KERNEL_ADALN, st);
}

// pos_major: out [n][pairs] (the zi_rope_table layout); else [pairs][n] for the QKV epilogue.
int run_rope(const zi_config& cfg, const int32_t* pos, int n, float2* out, cudaStream_t st, bool pos_major) {
  const int pairs = cfg.head_dim / 2;
  const int total = n * pairs;
  prof_pre(st);
  rope_table_kernel<<<(total + 255) / 256, 256, 0, st>>>(pos, n, cfg.rope_axes[0], cfg.rope_axes[1],
                                                           cfg.rope_axes[2], double(cfg.rope_theta), out,
                                                           pos_major ? 1 : 0);
  return launched(ZI_KERNEL_ROPE, st);
}

// Elementwise 2^x through the attention softmax's FMA-pipe exponential (exp2_poly_pair),
// for the test hook zi_exp2_poly.
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, size_t n) {
  const size_t i = 2 * (size_t(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const bool two = i + 1 < n;
  float e0, e1;
  exp2_poly_pair(x[i], two ? x[i + 1] : 0.f, e0, e1);
  y[i] = e0;
  if (two) y[i + 1] = e1;
}

// ---------------------------------------------------------------- fixed scratch
// Scratch of zi_block_forward_noalloc: a file-scope device array, so the entry
// point needs no caller workspace and allocates nothing.  Host code must not use
// the symbol as a pointer (on the host it names a stand-in object, not device
// memory); the device address is looked up once per device with that device
// current and cached.
static __device__ __align__(256) unsigned char g_zi_static_scratch[ZI_STATIC_SCRATCH_BYTES];

void* g_scratch_addr[kMaxDevices] = {};

int static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZI_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_zi_static_scratch) != cudaSuccess || !p) return ZI_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return ZI_OK;
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

const char* zi_status_string(int s) {
  switch (s) {
    case ZI_OK: return "ok";
    case ZI_ERR_ARG: return "invalid argument";
    case ZI_ERR_SHAPE: return "unsupported shape";
    case ZI_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
    case ZI_ERR_WORKSPACE: return "workspace missing or too small";
    case ZI_ERR_CUDA: return "CUDA call failed";
    case ZI_ERR_TIMEOUT: return "device pipeline wait timed out";
    case ZI_ERR_DEVICE: return "current device is not an sm_100 GPU";
    case ZI_ERR_SCRATCH_LIMIT: return "sizes exceed the library's fixed scratch (ZI_STATIC_SCRATCH_BYTES)";
    default: return "unknown status";
  }
}

int zi_version(void) { return kVersion; }

int zi_config_default(zi_config* c) {
  if (!c) return ZI_ERR_ARG;
  c->dim = 3840;
  c->heads = 30;
  c->head_dim = 128;
  c->ffn = 10240;
  c->cap_dim = 2560;
  c->t_freq = 256;
  c->t_mid = 1024;
  c->in_ch = 16;
  c->patch = 2;
  c->n_noise = 2;
  c->n_ctx = 2;
  c->n_main = 30;
  c->rope_axes[0] = 32;
  c->rope_axes[1] = 48;
  c->rope_axes[2] = 48;
  c->rope_theta = 256.0f;
  c->norm_eps = 1e-5f;
  c->final_eps = 1e-6f;
  c->t_scale = 1000.0f;
  return ZI_OK;
}

int zi_ffn_padded(int ffn) { return ffn <= 0 ? 0 : (ffn + 127) / 128 * 128; }

int zi_pack_qkv(const uint16_t* wq, const uint16_t* wk, const uint16_t* wv, int dim, uint16_t* w_qkv,
                zi_stream_t stream) {
  if (!wq || !wk || !wv || !w_qkv || dim <= 0) return ZI_ERR_ARG;
  const size_t n = size_t(dim) * dim * 2;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(w_qkv, wq, n, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(w_qkv + size_t(dim) * dim, wk, n, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(w_qkv + 2 * size_t(dim) * dim, wv, n, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return ZI_ERR_CUDA;
  return ZI_OK;
}

int zi_pack_ffn(const uint16_t* w1, const uint16_t* w3, const uint16_t* w2, int ffn, int dim, uint16_t* w13,
                uint16_t* w2p, zi_stream_t stream) {
  if (!w1 || !w3 || !w2 || !w13 || !w2p || ffn <= 0 || dim <= 0) return ZI_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int Fp = zi_ffn_padded(ffn);
  const size_t rowb = size_t(dim) * 2;
  if (Fp != ffn) {
    if (cudaMemsetAsync(w13, 0, size_t(2) * Fp * rowb, st) != cudaSuccess) return ZI_ERR_CUDA;
  }
  const int full = ffn / 128, tail = ffn % 128;
  // full 128-row groups: one strided copy per source
  if (full > 0) {
    if (cudaMemcpy2DAsync(w13, 256 * rowb, w1, 128 * rowb, 128 * rowb, full, cudaMemcpyDeviceToDevice, st) !=
            cudaSuccess ||
        cudaMemcpy2DAsync(w13 + 128 * size_t(dim), 256 * rowb, w3, 128 * rowb, 128 * rowb, full,
                          cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return ZI_ERR_CUDA;
  }
  if (tail > 0) {
    const size_t g = size_t(full);
    if (cudaMemcpyAsync(w13 + g * 256 * dim, w1 + g * 128 * dim, tail * rowb, cudaMemcpyDeviceToDevice, st) !=
            cudaSuccess ||
        cudaMemcpyAsync(w13 + (g * 256 + 128) * dim, w3 + g * 128 * dim, tail * rowb, cudaMemcpyDeviceToDevice,
                        st) != cudaSuccess)
      return ZI_ERR_CUDA;
  }
  if (Fp != ffn) {
    if (cudaMemsetAsync(w2p, 0, size_t(dim) * Fp * 2, st) != cudaSuccess) return ZI_ERR_CUDA;
  }
  if (cudaMemcpy2DAsync(w2p, size_t(Fp) * 2, w2, size_t(ffn) * 2, size_t(ffn) * 2, dim, cudaMemcpyDeviceToDevice,
                        st) != cudaSuccess)
    return ZI_ERR_CUDA;
  return ZI_OK;
}

int zi_block_workspace_size(const zi_config* cfg, int batch, int seq, size_t* h_bytes) {
  ZI_TRY(check_cfg(cfg));
  if (!h_bytes || batch <= 0 || seq <= 0) return ZI_ERR_ARG;
  *h_bytes = carve(*cfg, batch, seq, 0, false, 4 * cfg->dim).total;
  return ZI_OK;
}

int zi_model_workspace_size(const zi_config* cfg, int batch, int lat_h, int lat_w, int s_txt, size_t* h_bytes) {
  ZI_TRY(check_cfg(cfg));
  if (!h_bytes || batch <= 0 || lat_h <= 0 || lat_w <= 0 || s_txt <= 0) return ZI_ERR_ARG;
  if (lat_h % 2 || lat_w % 2) return ZI_ERR_SHAPE;
  const int s_img = (lat_h / 2) * (lat_w / 2);
  const int mod_cols = (cfg->n_noise + cfg->n_main) * 4 * cfg->dim + cfg->dim;
  *h_bytes = carve(*cfg, batch, s_img, s_txt, true, mod_cols).total;
  return ZI_OK;
}

int zi_positions(int s_txt, int grid_h, int grid_w, int32_t* d_pos, zi_stream_t stream) {
  if (!d_pos || s_txt < 0 || grid_h < 0 || grid_w < 0) return ZI_ERR_ARG;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  const int n = grid_h * grid_w + s_txt;
  if (n == 0) return ZI_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  prof_pre(st);
  positions_kernel<<<(n + 255) / 256, 256, 0, st>>>(s_txt, grid_h, grid_w, d_pos);
  return launched(ZI_KERNEL_POSITIONS, st);
}

int zi_rope_table(const zi_config* cfg, const int32_t* d_pos, int n, float* d_cos_sin, zi_stream_t stream) {
  ZI_TRY(check_cfg(cfg));
  if (!d_pos || !d_cos_sin || n < 0) return ZI_ERR_ARG;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  if (n == 0) return ZI_OK;
  return run_rope(*cfg, d_pos, n, reinterpret_cast<float2*>(d_cos_sin), reinterpret_cast<cudaStream_t>(stream),
                  true);
}

int zi_gemm_bf16(const uint16_t* d_a, const uint16_t* d_b, uint16_t* d_c, int m, int n, int k, zi_stream_t stream) {
  if (!d_a || !d_b || !d_c || m < 0 || n <= 0 || k <= 0) return ZI_ERR_ARG;
  if (!aligned16(d_a) || !aligned16(d_b) || !aligned16(d_c)) return ZI_ERR_ALIGN;
  if (k % 64 || n % 256) return ZI_ERR_SHAPE;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  return run_gemm<256, EPI_BF16>(dev, BIT_GEMM_BF16, ZI_KERNEL_GEMM, d_a, d_b, m, n, k, epi_plain(d_c, n),
                                 reinterpret_cast<cudaStream_t>(stream));
}

int zi_gemm_bf16_pair(const uint16_t* d_a, const uint16_t* d_b, uint16_t* d_c, int m, int n, int k,
                      zi_stream_t stream) {
  if (!d_a || !d_b || !d_c || m < 0 || n <= 0 || k <= 0) return ZI_ERR_ARG;
  if (!aligned16(d_a) || !aligned16(d_b) || !aligned16(d_c)) return ZI_ERR_ALIGN;
  if (k % 64 || n % 256) return ZI_ERR_SHAPE;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  return run_gemm_pair<EPI_BF16>(dev, BIT_GEMM_BF16, ZI_KERNEL_GEMM, d_a, d_b, m, n, k, epi_plain(d_c, n),
                                 reinterpret_cast<cudaStream_t>(stream));
}

int zi_quantize_rows_e4m3(const void* d_x, int x_bf16, int rows, int cols, uint8_t* d_q, float* d_s,
                          zi_stream_t stream) {
  if (!d_x || !d_q || !d_s || rows < 0 || cols <= 0 || (x_bf16 != 0 && x_bf16 != 1)) return ZI_ERR_ARG;
  if (cols % 4 || cols > kQuantMaxCols) return ZI_ERR_SHAPE;
  if (!aligned16(d_x) || !aligned16(d_q) || !aligned16(d_s)) return ZI_ERR_ALIGN;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (x_bf16) return run_quantize(static_cast<const uint16_t*>(d_x), rows, cols, d_q, d_s, st);
  return run_quantize(static_cast<const float*>(d_x), rows, cols, d_q, d_s, st);
}

int zi_gemm_e4m3(const uint8_t* d_a, const float* d_sa, const uint8_t* d_b, const float* d_sb, uint16_t* d_c, int m,
                 int n, int k, zi_stream_t stream) {
  if (!d_a || !d_sa || !d_b || !d_sb || !d_c || m < 0 || n <= 0 || k <= 0) return ZI_ERR_ARG;
  if (!aligned16(d_a) || !aligned16(d_b) || !aligned16(d_c) || !aligned16(d_sa) || !aligned16(d_sb))
    return ZI_ERR_ALIGN;
  if (k % 128 || n % 256) return ZI_ERR_SHAPE;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  EpiParams ep = epi_plain(d_c, n);
  ep.a_scale = d_sa;
  ep.b_scale = d_sb;
  return run_gemm<256, EPI_BF16, true>(dev, BIT_GEMM_BF16, ZI_KERNEL_GEMM, d_a, d_b, m, n, k, ep,
                                       reinterpret_cast<cudaStream_t>(stream));
}

int zi_attention(const uint16_t* d_qkv, uint16_t* d_out, int batch, int seq, int heads, zi_stream_t stream) {
  if (!d_qkv || !d_out || batch <= 0 || seq <= 0 || heads <= 0) return ZI_ERR_ARG;
  if (!aligned16(d_qkv) || !aligned16(d_out)) return ZI_ERR_ALIGN;
  if (heads > 65535 || batch > 65535) return ZI_ERR_SHAPE;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  const int row0[1] = {0}, len[1] = {seq};
  return run_attention(dev, d_qkv, batch * seq, d_out, heads * 128, heads, batch, 1, row0, len, nullptr,
                       reinterpret_cast<cudaStream_t>(stream));
}

int zi_attention_varlen(const uint16_t* d_qkv, uint16_t* d_out, int batch, int seq, int heads,
                        const int32_t* d_kv_len, zi_stream_t stream) {
  if (!d_qkv || !d_out || !d_kv_len || batch <= 0 || seq <= 0 || heads <= 0) return ZI_ERR_ARG;
  if (!aligned16(d_qkv) || !aligned16(d_out) || (reinterpret_cast<uintptr_t>(d_kv_len) & 3u)) return ZI_ERR_ALIGN;
  if (heads > 65535 || batch > 65535) return ZI_ERR_SHAPE;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  const int row0[1] = {0}, len[1] = {seq};
  return run_attention(dev, d_qkv, batch * seq, d_out, heads * 128, heads, batch, 1, row0, len, d_kv_len,
                       reinterpret_cast<cudaStream_t>(stream));
}

int zi_block_forward(const zi_config* cfg, const zi_block_weights* w, const float* d_c, const int32_t* d_pos,
                     int batch, int seq, const float* d_x_in, float* d_x_out, void* d_ws, size_t ws_bytes,
                     zi_stream_t stream) {
  ZI_TRY(check_cfg(cfg));
  if (!w || !d_pos || !d_x_in || !d_x_out || batch <= 0 || seq <= 0) return ZI_ERR_ARG;
  const bool modulated = w->w_ada != nullptr;
  if (!block_ptrs_ok(w, false) || (modulated && !d_c)) return ZI_ERR_ARG;
  if (!block_align_ok(w) || !aligned16(d_x_in) || !aligned16(d_x_out) || (d_c && !aligned16(d_c)))
    return ZI_ERR_ALIGN;
  if (size_t(batch) * seq > (size_t(1) << 30) || batch > 65535) return ZI_ERR_SHAPE;
  const Ws L = carve(*cfg, batch, seq, 0, false, 4 * cfg->dim);
  if (!d_ws || ws_bytes < L.total) return ZI_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(d_ws) & 255u) return ZI_ERR_ALIGN;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(d_ws);
  const int D = cfg->dim;
  const int rows = batch * seq;
  float* mod = reinterpret_cast<float*>(ws + L.mod);
  float2* rope = reinterpret_cast<float2*>(ws + L.rope);

  if (modulated) {
    AdaSegs segs;
    memset(&segs, 0, sizeof(segs));
    segs.n = 1;
    segs.w[0] = w->w_ada;
    segs.b[0] = w->b_ada;
    segs.rows[0] = 4 * D;
    segs.off[0] = 0;
    segs.dim = D;
    ZI_TRY(run_ada(segs, d_c, d_c, batch, 4 * D, mod, st));
  }
  ZI_TRY(run_rope(*cfg, d_pos, seq, rope, st, false));

  BlockCtx b;
  b.dev = dev;
  b.cfg = cfg;
  b.w = w;
  b.rows = rows;
  b.row_off = 0;
  b.batch = batch;
  b.map = RowMap{rows, seq, 1, 0};
  b.x_in = const_cast<float*>(d_x_in);
  b.x_out = d_x_out;
  b.h = reinterpret_cast<uint16_t*>(ws + L.h);
  b.hq = ws + L.h;
  b.hs = reinterpret_cast<float*>(ws + L.hs);
  b.q8 = ws + L.q8;
  b.q8s = reinterpret_cast<float*>(ws + L.q8s);
  b.qkv = reinterpret_cast<uint16_t*>(ws + L.qkv);
  b.att = reinterpret_cast<uint16_t*>(ws + L.att);
  b.o = reinterpret_cast<uint16_t*>(ws + L.o);
  b.u = reinterpret_cast<uint16_t*>(ws + L.u);
  b.rope = rope;
  b.rope_n = seq;
  b.mod = modulated ? mod : nullptr;
  b.mod_ld = 4 * D;
  b.nseg = 1;
  b.seg_row0[0] = 0;
  b.seg_len[0] = seq;
  b.seg_row0[1] = 0;
  b.seg_len[1] = 1;
  b.kv_len = nullptr;
  b.split = SplitScratch{reinterpret_cast<float4*>(ws + L.split_part), reinterpret_cast<int*>(ws + L.split_cnt)};
  ZI_TRY(clear_split(b.split, st));
  const bool f8 = block_f8(w);
  ZI_TRY(run_rms_mod<float>(d_x_in, rows, D, w->g_attn1, b.mod, b.mod_ld, b.map, 0, cfg->norm_eps, b.h, st,
                            f8 ? b.hq : nullptr, f8 ? b.hs : nullptr));
  const NextNormSpec none{NEXT_NONE, nullptr, nullptr, 0};
  return run_block(b, none, st);
}

int zi_block_forward_noalloc(const zi_config* cfg, const zi_block_weights* w, const float* d_c,
                             const int32_t* d_pos, int batch, int seq, const float* d_x_in, float* d_x_out,
                             zi_stream_t stream) {
  ZI_TRY(check_cfg(cfg));
  if (batch <= 0 || seq <= 0) return ZI_ERR_ARG;
  if (size_t(batch) * seq > (size_t(1) << 30)) return ZI_ERR_SHAPE;
  if (carve(*cfg, batch, seq, 0, false, 4 * cfg->dim).total > size_t(ZI_STATIC_SCRATCH_BYTES))
    return ZI_ERR_SCRATCH_LIMIT;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  void* ws = nullptr;
  ZI_TRY(static_scratch(&ws));
  return zi_block_forward(cfg, w, d_c, d_pos, batch, seq, d_x_in, d_x_out, ws, size_t(ZI_STATIC_SCRATCH_BYTES),
                          stream);
}

namespace {
int model_forward_impl(const zi_config* cfg, const zi_model_weights* w, int batch, int lat_h, int lat_w, int s_txt,
                       const int32_t* h_txt_len, const float* d_latent, const float* d_t, const uint16_t* d_txt,
                       float* d_out, float* d_trace, void* d_ws, size_t ws_bytes, zi_stream_t stream) {
  ZI_TRY(check_cfg(cfg));
  if (!w || !d_latent || !d_t || !d_txt || !d_out || batch <= 0 || lat_h <= 0 || lat_w <= 0 || s_txt <= 0)
    return ZI_ERR_ARG;
  if (h_txt_len) {
    if (!w->cap_pad) return ZI_ERR_ARG;
    for (int b = 0; b < batch; ++b)
      if (h_txt_len[b] < 1 || h_txt_len[b] > s_txt) return ZI_ERR_ARG;
  }
  if (lat_h % 2 || lat_w % 2) return ZI_ERR_SHAPE;
  if (batch > 65535) return ZI_ERR_SHAPE;
  const void* top[] = {w->x_emb_w, w->x_emb_b, w->cap_norm, w->cap_w, w->cap_b, w->t_w1, w->t_b1, w->t_w2,
                       w->t_b2, w->final_ada_w, w->final_ada_b, w->final_w, w->final_b};
  for (const void* p : top)
    if (!p) return ZI_ERR_ARG;
  if ((cfg->n_noise && !w->noise) || (cfg->n_ctx && !w->ctx) || !w->main) return ZI_ERR_ARG;
  for (int i = 0; i < cfg->n_noise; ++i)
    if (!block_ptrs_ok(&w->noise[i], true) || !block_align_ok(&w->noise[i])) return ZI_ERR_ARG;
  for (int i = 0; i < cfg->n_ctx; ++i)
    if (!block_ptrs_ok(&w->ctx[i], false) || w->ctx[i].w_ada || !block_align_ok(&w->ctx[i])) return ZI_ERR_ARG;
  for (int i = 0; i < cfg->n_main; ++i)
    if (!block_ptrs_ok(&w->main[i], true) || !block_align_ok(&w->main[i])) return ZI_ERR_ARG;
  // every block in e4m3 or none (the blocks hand their normalised input h to each other)
  const bool f8 = block_f8(&w->main[0]);
  for (int i = 0; i < cfg->n_noise; ++i)
    if (block_f8(&w->noise[i]) != f8) return ZI_ERR_ARG;
  for (int i = 0; i < cfg->n_ctx; ++i)
    if (block_f8(&w->ctx[i]) != f8) return ZI_ERR_ARG;
  for (int i = 0; i < cfg->n_main; ++i)
    if (block_f8(&w->main[i]) != f8) return ZI_ERR_ARG;
  const bool f8all = block_f8_all(&w->main[0]);
  for (int i = 0; i < cfg->n_noise; ++i)
    if (block_f8_all(&w->noise[i]) != f8all) return ZI_ERR_ARG;
  for (int i = 0; i < cfg->n_ctx; ++i)
    if (block_f8_all(&w->ctx[i]) != f8all) return ZI_ERR_ARG;
  for (int i = 0; i < cfg->n_main; ++i)
    if (block_f8_all(&w->main[i]) != f8all) return ZI_ERR_ARG;
  if (!aligned16(w->x_emb_w) || !aligned16(w->cap_w) || !aligned16(w->final_w) || !aligned16(w->final_ada_w) ||
      !aligned16(w->x_emb_b) || !aligned16(w->cap_b) || !aligned16(w->cap_norm) || !aligned16(d_txt) ||
      !aligned16(d_latent) || !aligned16(d_out))
    return ZI_ERR_ALIGN;

  const int D = cfg->dim;
  const int gh = lat_h / 2, gw = lat_w / 2;
  const int s_img = gh * gw;
  const int S = s_img + s_txt;
  const int rows_img = batch * s_img, rows_txt = batch * s_txt, rows = rows_img + rows_txt;
  const int n_mod = cfg->n_noise + cfg->n_main;
  const int mod_ld = n_mod * 4 * D + D;
  const Ws L = carve(*cfg, batch, s_img, s_txt, true, mod_ld);
  if (!d_ws || ws_bytes < L.total) return ZI_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(d_ws) & 255u) return ZI_ERR_ALIGN;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(d_ws);
  float* mod = reinterpret_cast<float*>(ws + L.mod);
  float* c = reinterpret_cast<float*>(ws + L.c);
  float* silu_c = reinterpret_cast<float*>(ws + L.silu);
  int32_t* pos = reinterpret_cast<int32_t*>(ws + L.pos);
  float2* rope = reinterpret_cast<float2*>(ws + L.rope);
  float* x = reinterpret_cast<float*>(ws + L.x);
  uint16_t* h = reinterpret_cast<uint16_t*>(ws + L.h);
  float* hs = reinterpret_cast<float*>(ws + L.hs);
  uint16_t* qkv = reinterpret_cast<uint16_t*>(ws + L.qkv);
  uint16_t* att = reinterpret_cast<uint16_t*>(ws + L.att);
  uint16_t* o = reinterpret_cast<uint16_t*>(ws + L.o);
  uint16_t* u = reinterpret_cast<uint16_t*>(ws + L.u);
  uint16_t* tok = reinterpret_cast<uint16_t*>(ws + L.tok);
  uint16_t* capn = reinterpret_cast<uint16_t*>(ws + L.capn);
  int* lens = h_txt_len ? reinterpret_cast<int*>(ws + L.lens) : nullptr;
  const RowMap map{rows_img, s_img, s_txt, h_txt_len ? S : 0};
  const SplitScratch split{reinterpret_cast<float4*>(ws + L.split_part), reinterpret_cast<int*>(ws + L.split_cnt)};
  const float eps = cfg->norm_eps;
  int traced = 0;
  auto trace = [&]() -> int {
    if (!d_trace) return ZI_OK;
    const size_t n = size_t(rows) * D;
    if (cudaMemcpyAsync(d_trace + size_t(traced++) * n, x, n * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return ZI_ERR_CUDA;
    return ZI_OK;
  };

  ZI_TRY(clear_split(split, st));
  // timestep conditioning and every adaLN projection
  {
    float* hid = reinterpret_cast<float*>(ws + L.hid);
    prof_pre(st);
    temb_hidden_kernel<<<dim3((cfg->t_mid + 7) / 8, batch), 256, 0, st>>>(d_t, cfg->t_scale, cfg->t_mid, w->t_w1,
                                                                         w->t_b1, hid);
    ZI_TRY(launched(ZI_KERNEL_TIMESTEP, st));
    prof_pre(st);
    temb_out_kernel<<<dim3(256 / 8, batch), 256, 0, st>>>(hid, cfg->t_mid, 256, w->t_w2, w->t_b2, c, silu_c);
    ZI_TRY(launched(ZI_KERNEL_TIMESTEP, st));
    AdaSegs segs;
    memset(&segs, 0, sizeof(segs));
    int k = 0;
    for (int i = 0; i < cfg->n_noise; ++i, ++k) {
      segs.w[k] = w->noise[i].w_ada;
      segs.b[k] = w->noise[i].b_ada;
      segs.rows[k] = 4 * D;
      segs.off[k] = k * 4 * D;
    }
    for (int i = 0; i < cfg->n_main; ++i, ++k) {
      segs.w[k] = w->main[i].w_ada;
      segs.b[k] = w->main[i].b_ada;
      segs.rows[k] = 4 * D;
      segs.off[k] = k * 4 * D;
    }
    segs.w[k] = w->final_ada_w;
    segs.b[k] = w->final_ada_b;
    segs.rows[k] = D;
    segs.off[k] = n_mod * 4 * D;
    segs.final_seg[k] = 1;
    segs.n = k + 1;
    segs.dim = D;
    ZI_TRY(run_ada(segs, c, silu_c, batch, mod_ld, mod, st));
  }
  auto mod_of_noise = [&](int i) { return mod + size_t(i) * 4 * D; };
  auto mod_of_main = [&](int i) { return mod + size_t(cfg->n_noise + i) * 4 * D; };
  const float* final_scale = mod + size_t(n_mod) * 4 * D;

  // positions and RoPE table: one sequence [image; text] shared by the batch, or,
  // with text lengths, one per element (its image positions follow its length)
  if (!h_txt_len) {
    prof_pre(st);
    positions_kernel<<<(S + 255) / 256, 256, 0, st>>>(s_txt, gh, gw, pos);
    ZI_TRY(launched(ZI_KERNEL_POSITIONS, st));
    ZI_TRY(run_rope(*cfg, pos, S, rope, st, false));
  } else {
    for (int b0 = 0; b0 < batch; b0 += kLenChunk) {
      LenChunk ch;
      memset(&ch, 0, sizeof(ch));
      ch.n = batch - b0 < kLenChunk ? batch - b0 : kLenChunk;
      for (int i = 0; i < ch.n; ++i) ch.v[i] = h_txt_len[b0 + i];
      prof_pre(st);
      store_lengths_kernel<<<1, kLenChunk, 0, st>>>(ch, lens + b0);
      ZI_TRY(launched(ZI_KERNEL_POSITIONS, st));
    }
    const long long n = static_cast<long long>(rows);
    prof_pre(st);
    positions_varlen_kernel<<<unsigned((n + 255) / 256), 256, 0, st>>>(s_txt, gh, gw, lens, batch, pos);
    ZI_TRY(launched(ZI_KERNEL_POSITIONS, st));
    ZI_TRY(run_rope(*cfg, pos, rows, rope, st, false));
  }

  // embedders: image rows [0, rows_img), text rows [rows_img, rows)
  {
    const size_t n = size_t(rows_img) * 64;
    prof_pre(st);
    patchify_kernel<<<unsigned((n + 255) / 256), 256, 0, st>>>(d_latent, batch, cfg->in_ch, lat_h, lat_w, tok);
    ZI_TRY(launched(ZI_KERNEL_PATCHIFY, st));
    EpiParams ex = epi_plain(x, D);
    ex.bias = w->x_emb_b;
    ZI_TRY((run_gemm<256, EPI_F32_BIAS>(dev, BIT_GEMM_F32, ZI_KERNEL_GEMM_EMBED, tok, w->x_emb_w, rows_img, D, 64, ex, st)));
    ZI_TRY(run_rms_mod<uint16_t>(d_txt, rows_txt, cfg->cap_dim, w->cap_norm, nullptr, 0, map, rows_img, eps, capn,
                                 st));
    EpiParams ec = epi_plain(x + size_t(rows_img) * D, D);
    ec.bias = w->cap_b;
    ZI_TRY((run_gemm<256, EPI_F32_BIAS>(dev, BIT_GEMM_F32, ZI_KERNEL_GEMM_EMBED, capn, w->cap_w, rows_txt, D,
                                        cfg->cap_dim, ec, st, split)));
    if (h_txt_len) {
      prof_pre(st);
      text_pad_kernel<<<dim3(s_txt, batch), 256, 0, st>>>(x + size_t(rows_img) * D, s_txt, D, lens, w->cap_pad);
      ZI_TRY(launched(ZI_KERNEL_TEXT_PAD, st));
    }
  }

  BlockCtx base;
  base.dev = dev;
  base.cfg = cfg;
  base.batch = batch;
  base.map = map;
  base.rope = rope;
  base.rope_n = h_txt_len ? rows : S;  // one table per element with text lengths
  base.mod_ld = mod_ld;
  base.kv_len = lens;
  base.split = split;

  const int Fp_ = zi_ffn_padded(cfg->ffn);
  auto segment_ctx = [&](int row_off, int nrows, int seglen) {
    BlockCtx b = base;
    b.rows = nrows;
    b.row_off = row_off;
    b.x_in = x + size_t(row_off) * D;
    b.x_out = b.x_in;
    b.h = h + size_t(row_off) * D;
    b.hq = ws + L.h + size_t(row_off) * D;  // e4m3 rows are D bytes
    b.hs = hs + row_off;
    b.q8 = ws + L.q8 + size_t(row_off) * (Fp_ > D ? Fp_ : D);
    b.q8s = reinterpret_cast<float*>(ws + L.q8s) + row_off;
    b.qkv = qkv + size_t(row_off) * 3 * D;
    b.att = att + size_t(row_off) * D;
    b.o = o + size_t(row_off) * D;
    b.u = u + size_t(row_off) * zi_ffn_padded(cfg->ffn);
    b.nseg = 1;
    b.seg_row0[0] = 0;
    b.seg_len[0] = seglen;
    b.seg_row0[1] = 0;
    b.seg_len[1] = 1;
    return b;
  };
  const NextNormSpec to_main0{NEXT_RMS, w->main[0].g_attn1, mod_of_main(0), 0, f8};

  // noise refiners on the image rows (all keys are image tokens: no key mask)
  {
    BlockCtx b = segment_ctx(0, rows_img, s_img);
    b.kv_len = nullptr;
    if (cfg->n_noise > 0) {
      ZI_TRY(run_rms_mod<float>(b.x_in, rows_img, D, w->noise[0].g_attn1, mod_of_noise(0), mod_ld, map, 0, eps,
                                b.h, st, f8 ? b.hq : nullptr, b.hs));
      for (int i = 0; i < cfg->n_noise; ++i) {
        b.w = &w->noise[i];
        b.mod = mod_of_noise(i);
        NextNormSpec nx = to_main0;
        if (i + 1 < cfg->n_noise) nx = NextNormSpec{NEXT_RMS, w->noise[i + 1].g_attn1, mod_of_noise(i + 1), 0, f8};
        nx.next_rows = rows_img;
        ZI_TRY(run_block(b, nx, st));
        ZI_TRY(trace());
      }
    } else {
      ZI_TRY(run_rms_mod<float>(b.x_in, rows_img, D, w->main[0].g_attn1, mod_of_main(0), mod_ld, map, 0, eps, b.h,
                                st, f8 ? b.hq : nullptr, b.hs));
    }
  }
  // context refiners on the text rows (unmodulated)
  {
    BlockCtx b = segment_ctx(rows_img, rows_txt, s_txt);
    if (cfg->n_ctx > 0) {
      ZI_TRY(run_rms_mod<float>(b.x_in, rows_txt, D, w->ctx[0].g_attn1, nullptr, 0, map, rows_img, eps, b.h, st,
                                f8 ? b.hq : nullptr, b.hs));
      for (int i = 0; i < cfg->n_ctx; ++i) {
        b.w = &w->ctx[i];
        b.mod = nullptr;
        NextNormSpec nx = to_main0;
        if (i + 1 < cfg->n_ctx) nx = NextNormSpec{NEXT_RMS, w->ctx[i + 1].g_attn1, nullptr, 0, f8};
        nx.next_rows = rows_txt;
        ZI_TRY(run_block(b, nx, st));
        ZI_TRY(trace());
      }
    } else {
      ZI_TRY(run_rms_mod<float>(b.x_in, rows_txt, D, w->main[0].g_attn1, mod_of_main(0), mod_ld, map, rows_img, eps,
                                b.h, st, f8 ? b.hq : nullptr, b.hs));
    }
  }
  // main blocks on the joint sequence (two segments per batch element)
  {
    BlockCtx b = segment_ctx(0, rows, s_img);
    b.nseg = 2;
    b.seg_row0[0] = 0;
    b.seg_len[0] = s_img;
    b.seg_row0[1] = rows_img;
    b.seg_len[1] = s_txt;
    for (int i = 0; i < cfg->n_main; ++i) {
      b.w = &w->main[i];
      b.mod = mod_of_main(i);
      NextNormSpec nx{NEXT_LAYERNORM, nullptr, final_scale, rows_img};
      if (i + 1 < cfg->n_main) nx = NextNormSpec{NEXT_RMS, w->main[i + 1].g_attn1, mod_of_main(i + 1), rows, f8};
      ZI_TRY(run_block(b, nx, st));
      ZI_TRY(trace());
    }
  }
  // final layer: LayerNorm(1 + scale) is already in h (image rows); linear + bias + unpatchify
  {
    EpiParams ef = epi_plain(d_out, 0);
    ef.bias = w->final_b;
    ef.s_img = s_img;
    ef.grid_w = gw;
    ef.lat_c = cfg->in_ch;
    ef.lat_h = lat_h;
    ef.lat_w = lat_w;
    ZI_TRY((run_gemm<64, EPI_UNPATCH>(dev, BIT_GEMM_UNPATCH, ZI_KERNEL_GEMM_FINAL, h, w->final_w, rows_img,
                                      4 * cfg->in_ch, D, ef, st, split)));
  }
  return ZI_OK;
}

}  // namespace

int zi_model_forward(const zi_config* cfg, const zi_model_weights* w, int batch, int lat_h, int lat_w, int s_txt,
                     const float* d_latent, const float* d_t, const uint16_t* d_txt, float* d_out, void* d_ws,
                     size_t ws_bytes, zi_stream_t stream) {
  return model_forward_impl(cfg, w, batch, lat_h, lat_w, s_txt, nullptr, d_latent, d_t, d_txt, d_out, nullptr, d_ws,
                            ws_bytes, stream);
}

int zi_model_forward_varlen(const zi_config* cfg, const zi_model_weights* w, int batch, int lat_h, int lat_w,
                            int s_txt, const int32_t* h_txt_len, const float* d_latent, const float* d_t,
                            const uint16_t* d_txt, float* d_out, void* d_ws, size_t ws_bytes, zi_stream_t stream) {
  if (!h_txt_len) return ZI_ERR_ARG;
  return model_forward_impl(cfg, w, batch, lat_h, lat_w, s_txt, h_txt_len, d_latent, d_t, d_txt, d_out, nullptr, d_ws,
                            ws_bytes, stream);
}

int zi_model_forward_trace(const zi_config* cfg, const zi_model_weights* w, int batch, int lat_h, int lat_w,
                           int s_txt, const float* d_latent, const float* d_t, const uint16_t* d_txt, float* d_out,
                           float* d_trace, void* d_ws, size_t ws_bytes, zi_stream_t stream) {
  if (!d_trace) return ZI_ERR_ARG;
  if (!aligned16(d_trace)) return ZI_ERR_ALIGN;
  return model_forward_impl(cfg, w, batch, lat_h, lat_w, s_txt, nullptr, d_latent, d_t, d_txt, d_out, d_trace, d_ws,
                            ws_bytes, stream);
}

int zi_euler_step(float* d_x, const float* d_out_cond, const float* d_out_uncond, float guidance, double sigma,
                  double sigma_next, size_t n, zi_stream_t stream) {
  if (n == 0) return ZI_OK;  // nothing to do; the pointers of empty arrays may be NULL
  if (!d_x || !d_out_cond) return ZI_ERR_ARG;
  if ((n + 255) / 256 > size_t(0x7fffffff)) return ZI_ERR_SHAPE;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  const float dt = float(sigma_next - sigma);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  prof_pre(st);
  euler_kernel<<<unsigned((n + 255) / 256), 256, 0, st>>>(d_x, d_out_cond, d_out_uncond, guidance, dt, n);
  return launched(ZI_KERNEL_EULER, st);
}

int zi_sigmas(int n_steps, double shift, double* h_sigmas) {
  if (n_steps <= 0 || !h_sigmas || !(shift > 0.0)) return ZI_ERR_ARG;
  for (int i = 0; i < n_steps; ++i) {
    const double s = n_steps == 1 ? 1.0 : 1.0 + (1.0 / n_steps - 1.0) * double(i) / double(n_steps - 1);
    h_sigmas[i] = shift * s / (1.0 + (shift - 1.0) * s);
  }
  h_sigmas[n_steps] = 0.0;
  return ZI_OK;
}

int zi_timesteps(int n_steps, double shift, float* h_t) {
  if (n_steps <= 0 || !h_t || !(shift > 0.0)) return ZI_ERR_ARG;
  std::vector<double> sig(size_t(n_steps) + 1);
  ZI_TRY(zi_sigmas(n_steps, shift, sig.data()));
  for (int i = 0; i < n_steps; ++i) h_t[i] = float(1.0 - sig[size_t(i)]);
  return ZI_OK;
}

int zi_profile_begin(int capacity) {
  if (capacity <= 0) return ZI_ERR_ARG;
  if (g_prof.on) return ZI_ERR_ARG;
  Prof p;
  p.ev.resize(size_t(capacity) + 1);
  p.kind.assign(size_t(capacity), 0);
  for (auto& e : p.ev) {
    if (cudaEventCreate(&e) != cudaSuccess) {
      for (auto& f : p.ev)
        if (f) cudaEventDestroy(f);
      return ZI_ERR_CUDA;
    }
  }
  p.cap = capacity;
  p.on = true;
  g_prof = std::move(p);
  return ZI_OK;
}

int zi_profile_end(float* h_ms, int* h_kinds, int capacity, int* h_count) {
  if (!g_prof.on) return ZI_ERR_ARG;
  int st = ZI_OK;
  const int n = g_prof.n;
  if (h_count) *h_count = g_prof.overflow ? -1 : n;
  if (n > 0 && cudaEventSynchronize(g_prof.ev[n]) != cudaSuccess) st = ZI_ERR_CUDA;
  for (int i = 0; i < n && i < capacity && st == ZI_OK; ++i) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, g_prof.ev[i], g_prof.ev[i + 1]) != cudaSuccess) st = ZI_ERR_CUDA;
    if (h_ms) h_ms[i] = ms;
    if (h_kinds) h_kinds[i] = g_prof.kind[i];
  }
  for (auto& e : g_prof.ev) cudaEventDestroy(e);
  g_prof = Prof();
  return st;
}

int zi_watchdog_selftest(int limit_us, zi_stream_t stream) {
  if (limit_us < 1 || limit_us > 2000000) return ZI_ERR_ARG;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  prof_pre(st);
  watchdog_selftest_kernel<<<1, 32, 0, st>>>(static_cast<unsigned long long>(limit_us) * 1000ull);
  return launched(ZI_KERNEL_SELFTEST, st);
}

int zi_exp2_poly(const float* d_x, float* d_y, size_t n, zi_stream_t stream) {
  if (n == 0) return ZI_OK;
  if (!d_x || !d_y) return ZI_ERR_ARG;
  const size_t threads = (n + 1) / 2;
  if ((threads + 255) / 256 > size_t(0x7fffffff)) return ZI_ERR_SHAPE;
  DevInfo* dev;
  ZI_TRY(current_device(&dev));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  prof_pre(st);
  exp2_poly_kernel<<<unsigned((threads + 255) / 256), 256, 0, st>>>(d_x, d_y, n);
  return launched(ZI_KERNEL_EXP2_TEST, st);
}

int zi_device_status(int* h_code) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, zi::g_zi_error, sizeof(v)) != cudaSuccess) return ZI_ERR_CUDA;
  if (h_code) *h_code = int(v);
  return v ? ZI_ERR_TIMEOUT : ZI_OK;
}

int zi_clear_device_status(void) {
  const unsigned int z = 0;
  if (cudaMemcpyToSymbol(zi::g_zi_error, &z, sizeof(z)) != cudaSuccess) return ZI_ERR_CUDA;
  return cudaDeviceSynchronize() == cudaSuccess ? ZI_OK : ZI_ERR_CUDA;
}

}  // extern "C"
