// KV compression for CSA (overlapping 2m-token windows, stride m) and HCA
// (non-overlapping m'-token windows).
//
// DeepSeek-V4 paper summary (hyper.ai), section "Method": CSA compresses every m
// tokens of the KV cache into one entry using learnable compression weights and
// a position bias; HCA merges every m' >> m tokens into one entry without
// overlapping compression.  Per channel c of entry i with window start s:
//   alpha_j = softmax over in-range j of (w[c] x[j,c] + b[j - s, c]),
//   y[i,c]  = sum_j alpha_j x[j,c].
// The softmax runs in fp32: the per-channel maximum of the logits, then one
// exponential per element (or online, for windows of unknown length).
//
// A thread owns 8 channels (one 16-byte load per token row).  CSA windows of 8
// rows (m = 4, bf16 output): one thread per (entry, channel group), its rows'
// logits kept in registers.  Other short windows: one warp per entry.  HCA
// windows of 128 rows: 16 row subsets per channel group in one CTA per entry,
// their maxima and sums merged in shared memory; other long windows: 8 warps
// per entry with online softmax states merged in shared memory.
#include "common.cuh"
#include "host_util.h"

namespace csa {
namespace {

struct CompressParams {
  const __nv_bfloat16* x;  // [B, xrows, d]: row j holds the token at position xpos0 + j
  const float* w;
  const float* b;
  int64_t B, T, N;  // tokens at positions < T exist; N entries computed per sequence
  int64_t i0;       // index of the first entry computed
  int64_t xpos0, xrows;
  int64_t n_out;    // entries per sequence in the output (its row pitch)
  // packed documents (nullable): sequence s = tokens [cu_tok[s], cu_tok[s+1]) of
  // x (xrows = total tokens, B = 1) whose entries are out rows [cu_ent[s], cu_ent[s+1])
  const int32_t* cu_tok;
  const int32_t* cu_ent;
  int n_seqs;
  int d, G;  // channels and 8-channel groups
  int stride, cwin;
  int layout;
  void* out;
  __nv_bfloat16* out_rope;
  float* out_scale;
};

// Entry e of the launch -> (output row, entry index i in its sequence, x base
// pointer at position 0 of the sequence, tokens T of the sequence).
struct EntryRef {
  int64_t out_row, i, T;
  const __nv_bfloat16* x0;
};

// True when position j of the entry's sequence is a row of the raw buffer
// (checked builds only; the host validates the buffer's coverage).
__device__ __forceinline__ bool x_row_ok(const CompressParams& p, const EntryRef& er, int64_t j) {
  const int64_t row = (er.x0 - p.x) / p.d + j;
  return CSA_INBOUNDS(row >= 0 && row < p.B * p.xrows);
}
__device__ __forceinline__ EntryRef entry_ref(const CompressParams& p, int64_t e) {
  EntryRef r;
  if (p.cu_tok != nullptr) {
    const int s = seq_of(p.cu_ent, p.n_seqs, e);
    const int64_t t0 = __ldg(p.cu_tok + s);
    r.out_row = e;
    r.i = e - __ldg(p.cu_ent + s);
    r.T = __ldg(p.cu_tok + s + 1) - t0;
    r.x0 = p.x + t0 * p.d;
    return r;
  }
  const int64_t b = e / p.N;
  r.i = p.i0 + e % p.N;
  r.out_row = b * p.n_out + r.i;
  r.T = p.T;
  r.x0 = p.x + (b * p.xrows - p.xpos0) * p.d;
  return r;
}

struct Acc8 {
  float m[8], s[8], a[8];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      m[c] = -INFINITY;
      s[c] = 0.f;
      a[c] = 0.f;
    }
  }
  __device__ __forceinline__ void add(const float* xv, const float* wv, const float* bv) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float l = fmaf(wv[c], xv[c], bv[c]);
      float mn = fmaxf(m[c], l);
      float corr = __expf(m[c] - mn);
      float p = __expf(l - mn);
      s[c] = fmaf(s[c], corr, p);
      a[c] = fmaf(a[c], corr, p * xv[c]);
      m[c] = mn;
    }
  }
};

__device__ __forceinline__ void unpack8(uint4 r, float* f) {
  f[0] = bf16_lo(r.x); f[1] = bf16_hi(r.x);
  f[2] = bf16_lo(r.y); f[3] = bf16_hi(r.y);
  f[4] = bf16_lo(r.z); f[5] = bf16_hi(r.z);
  f[6] = bf16_lo(r.w); f[7] = bf16_hi(r.w);
}

__device__ __forceinline__ void load8f(const float* p, float* f) {
  float4 u = __ldg(reinterpret_cast<const float4*>(p));
  float4 v = __ldg(reinterpret_cast<const float4*>(p + 4));
  f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
  f[4] = v.x; f[5] = v.y; f[6] = v.z; f[7] = v.w;
}

// 2^x by the hardware approximation (relative error ~2^-22, far below the
// bf16 rounding of the entry it weights); 0 for x = -inf.
__device__ __forceinline__ float exp2f_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Writes output row e.  Called by all 32 lanes; lane g < G holds channels
// [8g, 8g+8) in y.
__device__ __forceinline__ void store_entry(const CompressParams& p, int64_t e, int lane, const float* y) {
  if (p.layout == CSA_KV_BF16) {
    if (lane < p.G) {
      uint4 o;
      o.x = pack_bf16x2(y[0], y[1]);
      o.y = pack_bf16x2(y[2], y[3]);
      o.z = pack_bf16x2(y[4], y[5]);
      o.w = pack_bf16x2(y[6], y[7]);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + e * p.d + 8 * lane) = o;
    }
    return;
  }
  // split FP8 storage (d == 192): lanes 0..15 hold the 128 nope channels,
  // lanes 16..23 the 64 RoPE channels.
  float am = 0.f;
  if (lane < 16) {
#pragma unroll
    for (int c = 0; c < 8; ++c) am = fmaxf(am, fabsf(y[c]));
  }
#pragma unroll
  for (int o = 8; o; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const float scale = am > 0.f ? am / 448.0f : 1.0f;
  if (lane < 16) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int c = 0; c < 4; c += 2) {
      __nv_fp8x2_storage_t q0 =
          __nv_cvt_float2_to_fp8x2(make_float2(y[c] / scale, y[c + 1] / scale), __NV_SATFINITE, __NV_E4M3);
      lo |= static_cast<uint32_t>(q0) << (8 * c);
      __nv_fp8x2_storage_t q1 = __nv_cvt_float2_to_fp8x2(make_float2(y[c + 4] / scale, y[c + 5] / scale),
                                                         __NV_SATFINITE, __NV_E4M3);
      hi |= static_cast<uint32_t>(q1) << (8 * c);
    }
    *reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.out) + e * kDNope + 8 * lane) = make_uint2(lo, hi);
    if (lane == 0) p.out_scale[e] = scale;
  } else if (lane < 24) {
    uint4 o;
    o.x = pack_bf16x2(y[0], y[1]);
    o.y = pack_bf16x2(y[2], y[3]);
    o.z = pack_bf16x2(y[4], y[5]);
    o.w = pack_bf16x2(y[6], y[7]);
    *reinterpret_cast<uint4*>(p.out_rope + e * kDRope + 8 * (lane - 16)) = o;
  }
}

// One warp per entry (short windows).
__global__ void __launch_bounds__(256) compress_short_kernel(CompressParams p) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t e = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  if (e >= p.B * p.N) return;
  const EntryRef er = entry_ref(p, e);
  const int64_t start = er.i * p.stride - (p.cwin - p.stride);
  const int64_t j0 = start > 0 ? start : 0;
  const int64_t j1 = (start + p.cwin) < er.T ? (start + p.cwin) : er.T;
  float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (lane < p.G) {
    float wv[8];
    load8f(p.w + 8 * lane, wv);
    Acc8 acc;
    acc.init();
    const __nv_bfloat16* xb = er.x0 + 8 * lane;
    for (int64_t j = j0; j < j1; ++j) {
      float xv[8], bv[8];
      if (!x_row_ok(p, er, j)) continue;
      unpack8(ldg_nc16(xb + j * p.d), xv);
      load8f(p.b + (j - start) * p.d + 8 * lane, bv);
      acc.add(xv, wv, bv);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) y[c] = acc.a[c] / acc.s[c];
  }
  store_entry(p, er.out_row, lane, y);
}

// bf16 output, windows of CW rows known at compile time: one thread per
// (entry, 8-channel group), so every lane of every warp works whatever d is,
// and the CW row loads of a thread are all issued before the softmax runs.
// Consecutive threads read consecutive 16-byte chunks of a row.
template <int CW>
__global__ void __launch_bounds__(256) compress_flat_kernel(CompressParams p) {
  pdl_wait();
  pdl_trigger();
  const int64_t gidx = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int64_t n_ent = p.B * p.N;
  int64_t e;
  int g;
  EntryRef er;
  if (n_ent * p.G < (int64_t(1) << 31) && p.cu_tok == nullptr) {
    // every index below 2^31: 32-bit divisions (the 64-bit ones are emulated
    // and cost more than the entry's arithmetic)
    const uint32_t gi = static_cast<uint32_t>(gidx), G = static_cast<uint32_t>(p.G);
    const uint32_t e32 = gi / G;
    g = static_cast<int>(gi - e32 * G);
    e = e32;
    if (e >= n_ent) return;
    const uint32_t N = static_cast<uint32_t>(p.N), b = e32 / N;
    er.i = p.i0 + (e32 - b * N);
    er.out_row = static_cast<int64_t>(b) * p.n_out + er.i;
    er.T = p.T;
    er.x0 = p.x + (static_cast<int64_t>(b) * p.xrows - p.xpos0) * p.d;
  } else {
    e = gidx / p.G;
    g = static_cast<int>(gidx % p.G);
    if (e >= n_ent) return;
    er = entry_ref(p, e);
  }
  const int64_t start = er.i * p.stride - (CW - p.stride);
  float wv[8];
  load8f(p.w + 8 * g, wv);
  const __nv_bfloat16* xb = er.x0 + 8 * g;
  uint4 raw[CW];
#pragma unroll
  for (int r = 0; r < CW; ++r) {
    const int64_t j = start + r;
    raw[r] = (j >= 0 && j < er.T && x_row_ok(p, er, j)) ? ldg_nc16(xb + j * p.d) : make_uint4(0u, 0u, 0u, 0u);
  }
  // logits of every row kept in registers (rows outside the sequence take no
  // part: -inf), the per-channel maximum, then one exponential per element
  // with the subtraction folded into an FMA in the base-2 domain
  float lg[CW][8], mx[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) mx[c] = -INFINITY;
#pragma unroll
  for (int r = 0; r < CW; ++r) {
    const int64_t j = start + r;
    const bool in = j >= 0 && j < er.T;
    float xv[8], bv[8];
    unpack8(raw[r], xv);
    load8f(p.b + r * p.d + 8 * g, bv);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      lg[r][c] = in ? fmaf(wv[c], xv[c], bv[c]) : -INFINITY;
      mx[c] = fmaxf(mx[c], lg[r][c]);
    }
  }
  float sm[8], ac[8], m2[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    sm[c] = ac[c] = 0.f;
    m2[c] = mx[c] * kLog2e;
  }
#pragma unroll
  for (int r = 0; r < CW; ++r) {
    float xv[8];
    unpack8(raw[r], xv);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float ex = exp2f_fast(fmaf(lg[r][c], kLog2e, -m2[c]));  // 0 for rows outside the sequence
      sm[c] += ex;
      ac[c] = fmaf(ex, xv[c], ac[c]);
    }
  }
  uint4 o;
  o.x = pack_bf16x2(__fdividef(ac[0], sm[0]), __fdividef(ac[1], sm[1]));
  o.y = pack_bf16x2(__fdividef(ac[2], sm[2]), __fdividef(ac[3], sm[3]));
  o.z = pack_bf16x2(__fdividef(ac[4], sm[4]), __fdividef(ac[5], sm[5]));
  o.w = pack_bf16x2(__fdividef(ac[6], sm[6]), __fdividef(ac[7], sm[7]));
  *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + er.out_row * p.d + 8 * g) = o;
}

// Long windows of 128 rows (HCA with m' = 128): one CTA of 16 G threads per
// entry, thread (s, g) = 8 channels of group g over the 8 rows s, s + 16, ...;
// the per-channel maxima meet in shared memory first, then the partial sums,
// and warp 0 finishes the entry.  Every lane works whatever d is.
__global__ void __launch_bounds__(512) compress_wide_kernel(CompressParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[16][2][8][32];  // [row subset][max | sum, weighted sum][channel][group]
  const int tid = threadIdx.x;
  const int g = tid % p.G, rs = tid / p.G;
  const EntryRef er = entry_ref(p, blockIdx.x);
  const int64_t start = er.i * p.stride - (128 - p.stride);
  float wv[8];
  load8f(p.w + 8 * g, wv);
  const __nv_bfloat16* xb = er.x0 + 8 * g;
  uint4 raw[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t j = start + rs + 16 * i;
    raw[i] = (j >= 0 && j < er.T && x_row_ok(p, er, j)) ? ldg_nc16(xb + j * p.d) : make_uint4(0u, 0u, 0u, 0u);
  }
  float lg[8][8], mx[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) mx[c] = -INFINITY;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = rs + 16 * i;
    const int64_t j = start + r;
    const bool in = j >= 0 && j < er.T;
    float xv[8], bv[8];
    unpack8(raw[i], xv);
    load8f(p.b + r * p.d + 8 * g, bv);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      lg[i][c] = in ? fmaf(wv[c], xv[c], bv[c]) : -INFINITY;
      mx[c] = fmaxf(mx[c], lg[i][c]);
    }
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) red[rs][0][c][g] = mx[c];
  __syncthreads();
  float m2[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float m = -INFINITY;
#pragma unroll
    for (int s2 = 0; s2 < 16; ++s2) m = fmaxf(m, red[s2][0][c][g]);
    m2[c] = m == -INFINITY ? 0.f : m * kLog2e;
  }
  float sm[8], ac[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) sm[c] = ac[c] = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float xv[8];
    unpack8(raw[i], xv);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float ex = exp2f_fast(fmaf(lg[i][c], kLog2e, -m2[c]));
      sm[c] += ex;
      ac[c] = fmaf(ex, xv[c], ac[c]);
    }
  }
  __syncthreads();  // every thread has read the maxima
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    red[rs][0][c][g] = sm[c];
    red[rs][1][c][g] = ac[c];
  }
  __syncthreads();
  if (tid >= 32) return;
  const int lane = tid;
  float y[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float S = 0.f, A = 0.f;
    if (lane < p.G) {
#pragma unroll
      for (int s2 = 0; s2 < 16; ++s2) {
        S += red[s2][0][c][lane];
        A += red[s2][1][c][lane];
      }
    }
    y[c] = lane < p.G ? __fdividef(A, S) : 0.f;
  }
  store_entry(p, er.out_row, lane, y);
}

// One CTA per entry (long windows): 8 warps take interleaved rows, then warp 0
// merges the 8 partial softmax states.  RPW > 0: the window is 8 * RPW rows
// and each warp loads its RPW rows at once, then takes the maximum and one
// exponential per element; RPW == 0: any window, online softmax per row.
template <int RPW>
__global__ void __launch_bounds__(256) compress_long_kernel(CompressParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ float st[8][3][8][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const EntryRef er = entry_ref(p, blockIdx.x);
  const int64_t start = er.i * p.stride - (p.cwin - p.stride);
  const int64_t j0 = start > 0 ? start : 0;
  const int64_t j1 = (start + p.cwin) < er.T ? (start + p.cwin) : er.T;
  Acc8 acc;
  acc.init();
  if (lane < p.G) {
    float wv[8];
    load8f(p.w + 8 * lane, wv);
    const __nv_bfloat16* xb = er.x0 + 8 * lane;
    if constexpr (RPW > 0) {
      uint4 raw[RPW];
#pragma unroll
      for (int i = 0; i < RPW; ++i) {  // rows start + warp + 8 i, all loads in flight together
        const int64_t j = start + warp + 8 * i;
        raw[i] = (j >= j0 && j < j1 && x_row_ok(p, er, j)) ? ldg_nc16(xb + j * p.d) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        const int64_t j = start + warp + 8 * i;
        if (j < j0 || j >= j1) continue;
        float xv[8], bv[8];
        unpack8(raw[i], xv);
        load8f(p.b + (warp + 8 * i) * p.d + 8 * lane, bv);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc.m[c] = fmaxf(acc.m[c], fmaf(wv[c], xv[c], bv[c]));
      }
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        const int64_t j = start + warp + 8 * i;
        if (j < j0 || j >= j1) continue;
        float xv[8], bv[8];
        unpack8(raw[i], xv);
        load8f(p.b + (warp + 8 * i) * p.d + 8 * lane, bv);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float e = __expf(fmaf(wv[c], xv[c], bv[c]) - acc.m[c]);
          acc.s[c] += e;
          acc.a[c] = fmaf(e, xv[c], acc.a[c]);
        }
      }
    } else {
#pragma unroll 4
      for (int64_t j = j0 + warp; j < j1; j += 8) {
        float xv[8], bv[8];
        if (!x_row_ok(p, er, j)) continue;
        unpack8(ldg_nc16(xb + j * p.d), xv);
        load8f(p.b + (j - start) * p.d + 8 * lane, bv);
        acc.add(xv, wv, bv);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    st[warp][0][c][lane] = acc.m[c];
    st[warp][1][c][lane] = acc.s[c];
    st[warp][2][c][lane] = acc.a[c];
  }
  __syncthreads();
  if (warp != 0) return;
  float y[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) M = fmaxf(M, st[w][0][c][lane]);
    float S = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      float f = __expf(st[w][0][c][lane] - M);
      S = fmaf(st[w][1][c][lane], f, S);
      A = fmaf(st[w][2][c][lane], f, A);
    }
    y[c] = lane < p.G ? A / S : 0.f;
  }
  store_entry(p, er.out_row, lane, y);
}

csa_status check_args(const char* name, int32_t d, int32_t layout, const void* x, const float* w,
                      const float* b_pos, const void* out, const void* out_rope, const float* out_scale) {
  CSA_REQUIRE(d >= 8 && d <= 256 && d % 8 == 0, "%s: d must be a multiple of 8 in [8, 256] (got %d)", name, d);
  CSA_REQUIRE(layout == CSA_KV_BF16 || layout == CSA_KV_SPLIT_FP8, "%s: unknown out_layout %d", name, layout);
  if (layout == CSA_KV_SPLIT_FP8 && d != kDQK)
    return fail(CSA_ERR_UNSUPPORTED, "%s: split FP8 output needs d == 192 (got %d)", name, d);
  CSA_REQUIRE_PTR(x);
  CSA_REQUIRE_PTR(w);
  CSA_REQUIRE_PTR(b_pos);
  CSA_REQUIRE_PTR(out);
  if (layout == CSA_KV_SPLIT_FP8) {
    CSA_REQUIRE_PTR(out_rope);
    CSA_REQUIRE_PTR(out_scale);
  }
  return CSA_OK;
}

CompressParams base_params(const void* x, int32_t d, int32_t stride, int32_t cwin, const float* w,
                           const float* b_pos, int32_t layout, void* out, void* out_rope, float* out_scale) {
  CompressParams p;
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.w = w;
  p.b = b_pos;
  p.i0 = 0;
  p.xpos0 = 0;
  p.cu_tok = nullptr;
  p.cu_ent = nullptr;
  p.n_seqs = 0;
  p.d = d;
  p.G = d / 8;
  p.stride = stride;
  p.cwin = cwin;
  p.layout = layout;
  p.out = out;
  p.out_rope = static_cast<__nv_bfloat16*>(out_rope);
  p.out_scale = out_scale;
  return p;
}

csa_status launch(const char* name, const CompressParams& p, int64_t entries, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  prof_begin(s);
  cudaError_t e;
  if (p.layout == CSA_KV_BF16 && p.cwin == 8) {  // CSA with m = 4
    const int64_t threads = entries * p.G;
    e = launch_pdl(compress_flat_kernel<8>, dim3(static_cast<unsigned>((threads + 255) / 256)), dim3(256), 0, s, 1,
                   p);
  } else if (p.cwin <= 32) {
    e = launch_pdl(compress_short_kernel, dim3(static_cast<unsigned>((entries + 7) / 8)), dim3(256), 0, s, 1, p);
  } else if (p.cwin == 128) {  // HCA with m' = 128: 16 row subsets of 8 rows per channel group
    e = launch_pdl(compress_wide_kernel, dim3(static_cast<unsigned>(entries)), dim3(static_cast<unsigned>(16 * p.G)), 0,
                   s, 1, p);
  } else {
    e = launch_pdl(compress_long_kernel<0>, dim3(static_cast<unsigned>(entries)), dim3(256), 0, s, 1, p);
  }
  prof_end(s);
  return check_launch(name, e);
}

csa_status compress_impl(const char* name, const void* x, int64_t B, int64_t T, int32_t d, int32_t stride,
                         int32_t cwin, const float* w, const float* b_pos, int32_t layout, void* out,
                         void* out_rope, float* out_scale, void* stream) {
  clear_error();
  CSA_REQUIRE(B >= 0 && T >= 0 && B < (1LL << 31) && T < (1LL << 40), "%s: B must be in [0, 2^31), T in [0, 2^40)",
              name);
  if (B == 0 || T == 0) return CSA_OK;
  if (csa_status st = check_args(name, d, layout, x, w, b_pos, out, out_rope, out_scale); st != CSA_OK) return st;
  CompressParams p = base_params(x, d, stride, cwin, w, b_pos, layout, out, out_rope, out_scale);
  p.B = B;
  p.T = T;
  p.N = (T + stride - 1) / stride;
  p.xrows = T;
  p.n_out = p.N;
  CSA_REQUIRE(p.N < (1LL << 31) && B <= ((1LL << 31) - 1) / p.N, "%s: too many entries", name);
  return launch(name, p, B * p.N, stream);
}

// The entry completed by the token at position t (same t for every sequence of
// the call), from a buffer of recent raw tokens, written into a resident cache.
csa_status append_impl(const char* name, const void* x, int64_t B, int64_t rows, int64_t x_pos0, int64_t t,
                       int32_t d, int32_t stride, int32_t cwin, const float* w, const float* b_pos, int32_t layout,
                       void* out, void* out_rope, float* out_scale, int64_t n_cap, void* stream) {
  clear_error();
  CSA_REQUIRE(B >= 0 && B < (1LL << 31) && rows >= 0 && rows < (1LL << 40), "%s: bad B or rows", name);
  CSA_REQUIRE(t >= 0 && t < (1LL << 50) && x_pos0 >= 0, "%s: t and x_pos0 must be >= 0", name);
  CSA_REQUIRE(n_cap >= 0 && n_cap < (1LL << 31) && (B == 0 || n_cap <= ((1LL << 31) - 1) / B),
              "%s: bad cache capacity", name);
  if (B == 0 || (t + 1) % stride != 0) return CSA_OK;  // no entry completes at this token
  const int64_t i = (t + 1) / stride - 1;
  CSA_REQUIRE(i < n_cap, "%s: entry %lld does not fit a cache of %lld entries", name, static_cast<long long>(i),
              static_cast<long long>(n_cap));
  const int64_t start = i * stride - (cwin - stride);
  const int64_t lo = start > 0 ? start : 0;
  CSA_REQUIRE(x_pos0 <= lo && t - x_pos0 < rows,
              "%s: raw rows [%lld, %lld) do not hold the entry's tokens [%lld, %lld]", name,
              static_cast<long long>(x_pos0), static_cast<long long>(x_pos0 + rows), static_cast<long long>(lo),
              static_cast<long long>(t));
  if (csa_status st = check_args(name, d, layout, x, w, b_pos, out, out_rope, out_scale); st != CSA_OK) return st;
  CompressParams p = base_params(x, d, stride, cwin, w, b_pos, layout, out, out_rope, out_scale);
  p.B = B;
  p.T = t + 1;
  p.N = 1;
  p.i0 = i;
  p.xpos0 = x_pos0;
  p.xrows = rows;
  p.n_out = n_cap;
  return launch(name, p, B, stream);
}

// Packed sequences: each sequence of the packed buffer is compressed on its own.
csa_status packed_impl(const char* name, const void* x, const csa_packed* pk, int32_t d, int32_t stride,
                       int32_t cwin, const float* w, const float* b_pos, int32_t layout, void* out, void* out_rope,
                       float* out_scale, void* stream) {
  clear_error();
  CSA_REQUIRE(pk != nullptr, "%s: packed descriptor is NULL", name);
  CSA_REQUIRE(pk->n_seqs >= 0 && pk->total_tokens >= 0 && pk->total_tokens < (1LL << 31) &&
                  pk->total_entries >= 0 && pk->total_entries < (1LL << 31),
              "%s: bad packed descriptor sizes", name);
  if (pk->n_seqs == 0 || pk->total_entries == 0) return CSA_OK;
  CSA_REQUIRE(pk->cu_tokens != nullptr && pk->cu_entries != nullptr, "%s: packed offsets are NULL", name);
  if (csa_status st = check_args(name, d, layout, x, w, b_pos, out, out_rope, out_scale); st != CSA_OK) return st;
  CompressParams p = base_params(x, d, stride, cwin, w, b_pos, layout, out, out_rope, out_scale);
  p.B = 1;
  p.T = pk->total_tokens;
  p.N = pk->total_entries;
  p.xrows = pk->total_tokens;
  p.n_out = pk->total_entries;
  p.cu_tok = pk->cu_tokens;
  p.cu_ent = pk->cu_entries;
  p.n_seqs = pk->n_seqs;
  return launch(name, p, pk->total_entries, stream);
}

}  // namespace
}  // namespace csa

extern "C" {

csa_status csa_compress(const void* x, int64_t B, int64_t T, int32_t d, int32_t m, const float* w,
                        const float* b_pos, int32_t out_layout, void* out, void* out_rope, float* out_scale,
                        void* stream) {
  if (m < 1 || m > 64) return csa::fail(CSA_ERR_INVALID_ARG, "csa_compress: m must be in [1, 64] (got %d)", m);
  return csa::compress_impl("csa_compress", x, B, T, d, m, 2 * m, w, b_pos, out_layout, out, out_rope,
                            out_scale, stream);
}

csa_status hca_compress(const void* x, int64_t B, int64_t T, int32_t d, int32_t m_prime, const float* w,
                        const float* b_pos, int32_t out_layout, void* out, void* out_rope, float* out_scale,
                        void* stream) {
  if (m_prime < 1 || m_prime > 4096)
    return csa::fail(CSA_ERR_INVALID_ARG, "hca_compress: m' must be in [1, 4096] (got %d)", m_prime);
  return csa::compress_impl("hca_compress", x, B, T, d, m_prime, m_prime, w, b_pos, out_layout, out, out_rope,
                            out_scale, stream);
}

}  // extern "C"

namespace csa {
// Reads (and optionally clears) this unit's device error word.
CSA_DEFINE_DEVICE_ERROR_READER(compress_device_error)
}  // namespace csa

extern "C" {

csa_status csa_compress_append(const void* x, int64_t B, int64_t rows, int64_t x_pos0, int64_t t, int32_t d,
                               int32_t m, const float* w, const float* b_pos, int32_t out_layout, void* out,
                               void* out_rope, float* out_scale, int64_t n_cap, void* stream) {
  if (m < 1 || m > 64) return csa::fail(CSA_ERR_INVALID_ARG, "csa_compress_append: m must be in [1, 64] (got %d)", m);
  return csa::append_impl("csa_compress_append", x, B, rows, x_pos0, t, d, m, 2 * m, w, b_pos, out_layout, out,
                          out_rope, out_scale, n_cap, stream);
}

csa_status hca_compress_append(const void* x, int64_t B, int64_t rows, int64_t x_pos0, int64_t t, int32_t d,
                               int32_t m_prime, const float* w, const float* b_pos, int32_t out_layout, void* out,
                               void* out_rope, float* out_scale, int64_t n_cap, void* stream) {
  if (m_prime < 1 || m_prime > 4096)
    return csa::fail(CSA_ERR_INVALID_ARG, "hca_compress_append: m' must be in [1, 4096] (got %d)", m_prime);
  return csa::append_impl("hca_compress_append", x, B, rows, x_pos0, t, d, m_prime, m_prime, w, b_pos, out_layout,
                          out, out_rope, out_scale, n_cap, stream);
}

csa_status csa_compress_packed(const void* x, const csa_packed* packed, int32_t d, int32_t m, const float* w,
                               const float* b_pos, int32_t out_layout, void* out, void* out_rope, float* out_scale,
                               void* stream) {
  if (m < 1 || m > 64) return csa::fail(CSA_ERR_INVALID_ARG, "csa_compress_packed: m must be in [1, 64] (got %d)", m);
  return csa::packed_impl("csa_compress_packed", x, packed, d, m, 2 * m, w, b_pos, out_layout, out, out_rope,
                          out_scale, stream);
}

csa_status hca_compress_packed(const void* x, const csa_packed* packed, int32_t d, int32_t m_prime, const float* w,
                               const float* b_pos, int32_t out_layout, void* out, void* out_rope, float* out_scale,
                               void* stream) {
  if (m_prime < 1 || m_prime > 4096)
    return csa::fail(CSA_ERR_INVALID_ARG, "hca_compress_packed: m' must be in [1, 4096] (got %d)", m_prime);
  return csa::packed_impl("hca_compress_packed", x, packed, d, m_prime, m_prime, w, b_pos, out_layout, out, out_rope,
                          out_scale, stream);
}

}  // extern "C"
