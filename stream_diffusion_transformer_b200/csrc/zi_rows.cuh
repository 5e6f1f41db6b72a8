// Bandwidth-bound kernels: row norms with modulation and gated residuals,
// positions and the RoPE table, the timestep MLP, the batched adaLN GEMV,
// patchify, and the Euler / CFG step.  One CTA per row for the row kernels
// (256 threads, float4 / 8-byte bf16 vectors, every byte read once).
#pragma once
#include "zi_common.cuh"
#include "zi_gemm.cuh"

namespace zi {

constexpr int kRowThreads = 256;
constexpr int kRowMaxVec = 4;  // float4 per thread: rows up to 256 * 4 * 4 = 4096 wide

ZI_DEV float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();  // `red` may still be read from a previous reduction
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < kRowThreads / 32; ++i) t += red[i];
  return t;
}

ZI_DEV float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = red[0];
#pragma unroll
  for (int i = 1; i < kRowThreads / 32; ++i) t = fmaxf(t, red[i]);
  return t;
}

// Stores a row held by the CTA (y[k] for vector i = threadIdx.x + k * kRowThreads <
// nvec) as e4m3 codes with one fp32 scale: amax / 448, codes of y * (448 / amax)
// (round to nearest even, saturating); an all-zero row gets scale 1 and zero codes.
// Every thread of the CTA must call it.  MAXVEC: float4 per thread the row may need.
template <int MAXVEC = kRowMaxVec>
ZI_DEV void store_row_e4m3(const float4* y, int nvec, float* red, uint8_t* q, float* scale) {
  float m = 0.f;
#pragma unroll
  for (int k = 0; k < MAXVEC; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    if (i < nvec) m = fmaxf(m, fmaxf(fmaxf(fabsf(y[k].x), fabsf(y[k].y)), fmaxf(fabsf(y[k].z), fabsf(y[k].w))));
  }
  const float amax = block_max(m, red);
  const bool zero = amax == 0.f;
  const float inv = zero ? 0.f : __fdiv_rn(448.f, amax);
  if (threadIdx.x == 0) *scale = zero ? 1.f : __fdiv_rn(amax, 448.f);
#pragma unroll
  for (int k = 0; k < MAXVEC; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    if (i < nvec) {
      const float4 v = y[k];
      reinterpret_cast<uint32_t*>(q)[i] =
          zero ? 0u : pack_e4m3x4(__fmul_rn(v.x, inv), __fmul_rn(v.y, inv), __fmul_rn(v.z, inv), __fmul_rn(v.w, inv));
    }
  }
}

ZI_DEV float4 ld_bf16x4(const uint16_t* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xFFFF0000u));
}

ZI_DEV void st_bf16x4(uint16_t* p, float4 v) {
  uint2 u;
  u.x = pack_bf16x2(v.x, v.y);
  u.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(p) = u;
}

// h[row] = bf16( gain * x / sqrt(mean(x^2) + eps) * mscale[batch(row)] )
// x is fp32 (TIn = float) or bf16 (TIn = uint16_t); mscale holds 1 + scale as the
// adaLN kernel stores it, or is null (no modulation).  With hq non-null the row
// is written as e4m3 codes into hq [rows][D] with its scale in hs[row] instead.
template <typename TIn>
__global__ void __launch_bounds__(kRowThreads) rms_mod_kernel(const TIn* __restrict__ x, int D,
                                                              const uint16_t* __restrict__ gain,
                                                              const float* __restrict__ scale, int scale_ld,
                                                              RowMap map, int row_off, float eps,
                                                              uint16_t* __restrict__ h, uint8_t* __restrict__ hq,
                                                              float* __restrict__ hs) {
  __shared__ float red[kRowThreads / 32];
  const int row = blockIdx.x;
  const int nvec = D >> 2;
  float4 v[kRowMaxVec];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < kRowMaxVec; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < nvec) {
      if constexpr (sizeof(TIn) == 4) {
        v[k] = reinterpret_cast<const float4*>(x + size_t(row) * D)[i];
      } else {
        v[k] = ld_bf16x4(reinterpret_cast<const uint16_t*>(x) + size_t(row) * D + 4 * i);
      }
      ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
    }
  }
  const float r = rsqrtf(block_sum(ss, red) / float(D) + eps);
  const float* sc = scale ? scale + size_t(map.batch(row + row_off)) * scale_ld : nullptr;
#pragma unroll
  for (int k = 0; k < kRowMaxVec; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    if (i < nvec) {
      const float4 g = ld_bf16x4(gain + 4 * i);
      float4 m = make_float4(1.f, 1.f, 1.f, 1.f);
      if (sc) m = reinterpret_cast<const float4*>(sc)[i];
      v[k] = make_float4(v[k].x * r * g.x * m.x, v[k].y * r * g.y * m.y, v[k].z * r * g.z * m.z,
                         v[k].w * r * g.w * m.w);
      if (!hq) st_bf16x4(h + size_t(row) * D + 4 * i, v[k]);
    }
  }
  if (hq) store_row_e4m3(v, nvec, red, hq + size_t(row) * D, hs + row);
}

// Per-row e4m3 quantisation of x [rows][D] (fp32 or bf16): q [rows][D] codes and
// s [rows] scales, as store_row_e4m3 forms them.  One CTA per row; rows up to
// kRowThreads * MAXVEC * 4 wide.
template <typename TIn, int MAXVEC>
__global__ void __launch_bounds__(kRowThreads) quantize_rows_e4m3_kernel(const TIn* __restrict__ x, int D,
                                                                         uint8_t* __restrict__ q,
                                                                         float* __restrict__ s) {
  __shared__ float red[kRowThreads / 32];
  const int row = blockIdx.x;
  const int nvec = D >> 2;
  float4 v[MAXVEC];
#pragma unroll
  for (int k = 0; k < MAXVEC; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < nvec) {
      if constexpr (sizeof(TIn) == 4) {
        v[k] = reinterpret_cast<const float4*>(x + size_t(row) * D)[i];
      } else {
        v[k] = ld_bf16x4(reinterpret_cast<const uint16_t*>(x) + size_t(row) * D + 4 * i);
      }
    }
  }
  store_row_e4m3<MAXVEC>(v, nvec, red, q + size_t(row) * D, s + row);
}

enum NextNorm : int { NEXT_NONE = 0, NEXT_RMS = 1, NEXT_LAYERNORM = 2 };

// Gated residual with the post-sublayer RMSNorm, fused with the next sublayer's
// pre-norm:
//   x_out = x_in + gate * g_post * o / sqrt(mean(o^2) + eps)      (gate = tanh(raw) or 1)
//   h     = g_next * x_out / sqrt(mean(x_out^2) + eps) * (1 + scale)     (NEXT_RMS)
//   h     = (x_out - mean) / sqrt(var + eps_ln) * (1 + scale)            (NEXT_LAYERNORM)
// tanh(raw) and 1 + scale come precomputed from the adaLN kernel.
// h is written only for rows < next_rows.
struct PostParams {
  const float* x_in;
  float* x_out;
  const uint16_t* o;
  const uint16_t* g_post;
  const float* gate;  // tanh(gate) [B][gate_ld] or null (gate = 1)
  int gate_ld;
  int next;
  const uint16_t* g_next;  // NEXT_RMS gain
  const float* scale;      // 1 + scale [B][scale_ld] or null (no modulation)
  int scale_ld;
  int next_rows;
  uint16_t* h;
  uint8_t* hq;  // non-null: the next norm's output as e4m3 codes [rows][D] ...
  float* hs;    // ... with one scale per row (NEXT_RMS only)
  RowMap map;
  int row_off;  // global row of local row 0 (for the batch lookup)
  int D;
  float eps, eps_ln;
};

__global__ void __launch_bounds__(kRowThreads) post_residual_kernel(PostParams p) {
  __shared__ float red[kRowThreads / 32];
  const int row = blockIdx.x;
  const int D = p.D, nvec = D >> 2;
  const int b = p.map.batch(row + p.row_off);
  float4 v[kRowMaxVec], xv[kRowMaxVec];
  float ss = 0.f;
  // issue every load of the row (o and x) before the first reduction
#pragma unroll
  for (int k = 0; k < kRowMaxVec; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    xv[k] = v[k];
    if (i < nvec) {
      v[k] = ld_bf16x4(p.o + size_t(row) * D + 4 * i);
      xv[k] = reinterpret_cast<const float4*>(p.x_in + size_t(row) * D)[i];
    }
  }
#pragma unroll
  for (int k = 0; k < kRowMaxVec; ++k)
    ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
  const float ro = rsqrtf(block_sum(ss, red) / float(D) + p.eps);
  const float* gt = p.gate ? p.gate + size_t(b) * p.gate_ld : nullptr;
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int k = 0; k < kRowMaxVec; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    if (i < nvec) {
      const float4 x = xv[k];
      const float4 g = ld_bf16x4(p.g_post + 4 * i);
      float4 a = make_float4(1.f, 1.f, 1.f, 1.f);
      if (gt) a = reinterpret_cast<const float4*>(gt)[i];
      float4 y;
      y.x = x.x + a.x * g.x * (v[k].x * ro);
      y.y = x.y + a.y * g.y * (v[k].y * ro);
      y.z = x.z + a.z * g.z * (v[k].z * ro);
      y.w = x.w + a.w * g.w * (v[k].w * ro);
      reinterpret_cast<float4*>(p.x_out + size_t(row) * D)[i] = y;
      v[k] = y;
      s1 += y.x + y.y + y.z + y.w;
      s2 += y.x * y.x + y.y * y.y + y.z * y.z + y.w * y.w;
    }
  }
  if (p.next == NEXT_NONE || row >= p.next_rows) return;
  float mu = 0.f, r;
  if (p.next == NEXT_RMS) {
    r = rsqrtf(block_sum(s2, red) / float(D) + p.eps);
  } else {
    mu = block_sum(s1, red) / float(D);
    // variance from the centred values (second pass over registers)
    float sc = 0.f;
#pragma unroll
    for (int k = 0; k < kRowMaxVec; ++k) {
      const int i = threadIdx.x + k * kRowThreads;
      if (i < nvec) {
        const float a = v[k].x - mu, bq = v[k].y - mu, c = v[k].z - mu, d = v[k].w - mu;
        sc += a * a + bq * bq + c * c + d * d;
      }
    }
    r = rsqrtf(block_sum(sc, red) / float(D) + p.eps_ln);
  }
  const float* sc = p.scale ? p.scale + size_t(b) * p.scale_ld : nullptr;
#pragma unroll
  for (int k = 0; k < kRowMaxVec; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    if (i < nvec) {
      float4 g = make_float4(1.f, 1.f, 1.f, 1.f);
      if (p.next == NEXT_RMS) g = ld_bf16x4(p.g_next + 4 * i);
      float4 m = make_float4(1.f, 1.f, 1.f, 1.f);
      if (sc) m = reinterpret_cast<const float4*>(sc)[i];
      v[k] = make_float4((v[k].x - mu) * r * g.x * m.x, (v[k].y - mu) * r * g.y * m.y,
                         (v[k].z - mu) * r * g.z * m.z, (v[k].w - mu) * r * g.w * m.w);
      if (!p.hq) st_bf16x4(p.h + size_t(row) * D + 4 * i, v[k]);
    }
  }
  if (p.hq) store_row_e4m3(v, nvec, red, p.hq + size_t(row) * D, p.hs + row);
}

// Position ids of one sequence [image tokens; text tokens]:
// image token (r, c) -> (s_txt + 1, r, c); text token j -> (j + 1, 0, 0).
__global__ void positions_kernel(int s_txt, int grid_h, int grid_w, int* __restrict__ pos) {
  const int n_img = grid_h * grid_w;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n_img + s_txt) return;
  int a, b, c;
  if (t < n_img) {
    a = s_txt + 1;
    b = t / grid_w;
    c = t % grid_w;
  } else {
    a = t - n_img + 1;
    b = 0;
    c = 0;
  }
  pos[3 * t + 0] = a;
  pos[3 * t + 1] = b;
  pos[3 * t + 2] = c;
}

// Positions of a padded batch, one sequence per element b: [image; s_txt text
// rows], element b holding len[b] valid text tokens.  Image token (r, c) ->
// (len[b] + 1, r, c); text row j (valid or pad) -> (j + 1, 0, 0).  With the pad
// keys masked, this gives each element the positions of its unpadded sequence.
// pos int32 [batch][grid_h*grid_w + s_txt][3].
__global__ void positions_varlen_kernel(int s_txt, int grid_h, int grid_w, const int* __restrict__ len, int batch,
                                        int* __restrict__ pos) {
  const int n_img = grid_h * grid_w;
  const int S = n_img + s_txt;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<long long>(S) * batch) return;
  const int b = int(t / S), i = int(t % S);
  int a0, a1, a2;
  if (i < n_img) {
    a0 = len[b] + 1;
    a1 = i / grid_w;
    a2 = i % grid_w;
  } else {
    a0 = i - n_img + 1;
    a1 = 0;
    a2 = 0;
  }
  pos[3 * t + 0] = a0;
  pos[3 * t + 1] = a1;
  pos[3 * t + 2] = a2;
}

// Failure-detection self-test: one thread waits on an mbarrier that nothing
// arrives on; the bounded wait gives up after limit_ns, records
// ZI_DEVERR_TIMEOUT_SELFTEST in the device error word and the kernel returns.
__global__ void watchdog_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    mbar_wait(&bar, 0, &abort_flag, ZI_DEVERR_TIMEOUT_SELFTEST, limit_ns);
  }
}

__global__ void zero_ints_kernel(int* __restrict__ p, int n) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) p[i] = 0;
}

// Up to kLenChunk per-element text lengths carried by value into device memory
// (no host-to-device copy, so the forward stays capturable in a CUDA graph).
constexpr int kLenChunk = 64;
struct LenChunk {
  int n;
  int v[kLenChunk];
};

__global__ void store_lengths_kernel(LenChunk c, int* __restrict__ out) {
  if (int(threadIdx.x) < c.n) out[threadIdx.x] = c.v[threadIdx.x];
}

// Text rows j >= len[b] of element b take the cap_pad_token embedding (bf16 [D]).
// x_txt fp32 [batch][s_txt][D]; grid (s_txt, batch), 256 threads.
__global__ void text_pad_kernel(float* __restrict__ x_txt, int s_txt, int D, const int* __restrict__ len,
                                const uint16_t* __restrict__ pad) {
  const int j = blockIdx.x, b = blockIdx.y;
  if (j < len[b]) return;
  float* row = x_txt + (static_cast<size_t>(b) * s_txt + j) * D;
  for (int i = threadIdx.x; i < D; i += blockDim.x) row[i] = bf16_to_f32(pad[i]);
}

// (cos, sin) of pos[axis] * theta^(-2j/d_axis) for every token and rotation
// pair; pairs [0, a0/2) use axis 0, the next a1/2 axis 1, the last a2/2 axis 2.
// Angles are formed in fp64 and rounded to fp32 once.
// out[t][j] (pos_major) or out[j][t] (pair-major, the layout the QKV epilogue reads).
__global__ void rope_table_kernel(const int* __restrict__ pos, int n, int a0, int a1, int a2, double theta,
                                  float2* __restrict__ out, int pos_major) {
  const int pairs = (a0 + a1 + a2) / 2;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n * pairs) return;
  const int t = idx / pairs, j = idx % pairs;
  int axis, jj, da;
  if (j < a0 / 2) {
    axis = 0; jj = j; da = a0;
  } else if (j < (a0 + a1) / 2) {
    axis = 1; jj = j - a0 / 2; da = a1;
  } else {
    axis = 2; jj = j - (a0 + a1) / 2; da = a2;
  }
  const double omega = pow(theta, -2.0 * double(jj) / double(da));
  const double ang = double(pos[3 * t + axis]) * omega;
  double s, c;
  sincos(ang, &s, &c);
  out[pos_major ? idx : size_t(j) * n + t] = make_float2(float(c), float(s));
}

// Timestep conditioning, step 1: hid[b] = SiLU(W1 e + b1) with
// e = [cos(1000 t f_k), sin(1000 t f_k)], f_k = 10000^(-k/(t_freq/2)) (sinusoid in
// fp64).  grid (t_mid / 8, B), 256 threads: each CTA rebuilds e in smem, one warp
// per hidden unit with 16-byte weight loads (t_freq == 256: 8 inputs per lane).
__global__ void __launch_bounds__(256) temb_hidden_kernel(const float* __restrict__ t, float t_scale, int t_mid,
                                                          const uint16_t* __restrict__ w1,
                                                          const uint16_t* __restrict__ b1, float* __restrict__ hid) {
  __shared__ float e[256];
  const int b = blockIdx.y;
  const double tin = double(t[b]) * double(t_scale);
  for (int k = threadIdx.x; k < 128; k += blockDim.x) {
    const double f = exp(-log(10000.0) * double(k) / 128.0);
    double sn, co;
    sincos(tin * f, &sn, &co);
    e[k] = float(co);
    e[k + 128] = float(sn);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o = blockIdx.x * 8 + warp;
  if (o >= t_mid) return;
  const uint4 wv = *reinterpret_cast<const uint4*>(w1 + size_t(o) * 256 + lane * 8);
  const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
  float acc = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    acc = fmaf(__uint_as_float(ww[q] << 16), e[lane * 8 + 2 * q], acc);
    acc = fmaf(__uint_as_float(ww[q] & 0xFFFF0000u), e[lane * 8 + 2 * q + 1], acc);
  }
  acc = warp_sum(acc) + bf16_to_f32(b1[o]);
  if (lane == 0) hid[size_t(b) * t_mid + o] = acc / (1.0f + expf(-acc));
}

// Timestep conditioning, step 2: c[b] = W2 hid[b] + b2 (and SiLU(c) for the final
// layer's adaLN).  grid (ada / 8, B), one warp per output, 16-byte weight loads.
__global__ void __launch_bounds__(256) temb_out_kernel(const float* __restrict__ hid, int t_mid, int ada,
                                                       const uint16_t* __restrict__ w2,
                                                       const uint16_t* __restrict__ b2, float* __restrict__ c,
                                                       float* __restrict__ silu_c) {
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o = blockIdx.x * 8 + warp;
  if (o >= ada) return;
  const uint16_t* wr = w2 + size_t(o) * t_mid;
  const float* h = hid + size_t(b) * t_mid;
  float acc = 0.f;
  for (int i = lane * 8; i < t_mid; i += 256) {
    const uint4 wv = *reinterpret_cast<const uint4*>(wr + i);
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc = fmaf(__uint_as_float(ww[q] << 16), h[i + 2 * q], acc);
      acc = fmaf(__uint_as_float(ww[q] & 0xFFFF0000u), h[i + 2 * q + 1], acc);
    }
  }
  acc = warp_sum(acc) + bf16_to_f32(b2[o]);
  if (lane == 0) {
    c[size_t(b) * ada + o] = acc;
    silu_c[size_t(b) * ada + o] = acc / (1.0f + expf(-acc));
  }
}

// All adaLN projections of a forward in one launch, stored as the factors the
// row kernels multiply by.  A block segment (4D rows: scale_msa, gate_msa,
// scale_mlp, gate_mlp) maps c through w_s + b_s and stores 1 + scale and
// tanh(gate); the final layer's segment (D rows) maps SiLU(c) and stores
// 1 + scale.  out[b][off_s + row].  One warp per output row, 16-byte weight loads.
constexpr int kMaxAdaSegs = 40;
struct AdaSegs {
  const uint16_t* w[kMaxAdaSegs];
  const uint16_t* b[kMaxAdaSegs];
  int rows[kMaxAdaSegs];
  int off[kMaxAdaSegs];
  int final_seg[kMaxAdaSegs];  // 1: input SiLU(c), all rows are scales; 0: a block's 4 bands
  int n;
  int dim;
};

__global__ void __launch_bounds__(256) ada_gemv_kernel(AdaSegs segs, const float* __restrict__ c,
                                                       const float* __restrict__ silu_c, int batch, int out_ld,
                                                       float* __restrict__ out) {
  // ada width fixed at 256: each lane owns 8 consecutive inputs.
  const int s = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = segs.rows[s];
  const bool fin = segs.final_seg[s] != 0;
  const float* in = fin ? silu_c : c;
  for (int r = blockIdx.x * 8 + warp; r < rows; r += gridDim.x * 8) {
    const uint4 wv = *reinterpret_cast<const uint4*>(segs.w[s] + size_t(r) * 256 + lane * 8);
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
    float wf[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      wf[2 * q] = __uint_as_float(ww[q] << 16);
      wf[2 * q + 1] = __uint_as_float(ww[q] & 0xFFFF0000u);
    }
    const float bias = bf16_to_f32(segs.b[s][r]);
    const bool is_gate = !fin && ((r / segs.dim) & 1);  // bands 1 and 3 of a block are gates
    for (int b = 0; b < batch; ++b) {
      const float4 i0 = *reinterpret_cast<const float4*>(in + size_t(b) * 256 + lane * 8);
      const float4 i1 = *reinterpret_cast<const float4*>(in + size_t(b) * 256 + lane * 8 + 4);
      float acc = wf[0] * i0.x + wf[1] * i0.y + wf[2] * i0.z + wf[3] * i0.w + wf[4] * i1.x + wf[5] * i1.y +
                  wf[6] * i1.z + wf[7] * i1.w;
      acc = warp_sum(acc) + bias;
      if (lane == 0) out[size_t(b) * out_ld + segs.off[s] + r] = is_gate ? tanhf(acc) : 1.0f + acc;
    }
  }
}

// latent [B, C, H, W] fp32 -> tokens [B * (H/2)(W/2), 4C] bf16, feature (i*2 + j)*C + c.
__global__ void patchify_kernel(const float* __restrict__ lat, int B, int C, int H, int W,
                                uint16_t* __restrict__ tok) {
  const int gw = W / 2, gh = H / 2, F = 4 * C;
  const size_t total = size_t(B) * gh * gw * F;
  const size_t idx = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int f = int(idx % F);
  const size_t tkn = idx / F;
  const int b = int(tkn / (size_t(gh) * gw));
  const int t = int(tkn % (size_t(gh) * gw));
  const int r = t / gw, s = t % gw;
  const int c = f % C, pq = f / C;
  const float v = lat[((size_t(b) * C + c) * H + 2 * r + (pq >> 1)) * W + 2 * s + (pq & 1)];
  __nv_bfloat16 hb = __float2bfloat16_rn(v);
  tok[idx] = *reinterpret_cast<uint16_t*>(&hb);
}

// x += (sigma_next - sigma) * (-y),  y = out_u + g (out_c - out_u)  (or out_c without CFG).
__global__ void euler_kernel(float* __restrict__ x, const float* __restrict__ oc, const float* __restrict__ ou,
                             float g, float dt, size_t n) {
  const size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float y = oc[i];
  if (ou) y = ou[i] + g * (y - ou[i]);
  x[i] = x[i] + dt * (-y);
}

}  // namespace zi
