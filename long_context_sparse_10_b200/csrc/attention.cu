// Core attention of CSA (selected entries) and HCA (all visible entries), each
// joined with the sliding-window branch of raw recent tokens in ONE softmax.
//
// DeepSeek-V4 paper summary (hyper.ai), section "Method": CSA's core attention
// is multi-query attention with a single key/value head shared by all query
// heads, over the top-k compressed entries; HCA attends densely over all of its
// heavily compressed entries; both add a sliding-window attention branch.  The
// storage paragraph keeps RoPE channels in BF16 and the rest in FP8: with the
// split cache an entry's key is (e4m3 nope * scale) ++ rope and its value is
// the same scaled nope channels (shared key and value).
//
// One CTA (4 warps) handles one query row and a contiguous range of "key
// slots" (entry slots first, then window slots) in tiles of 64 keys staged in
// shared memory.  All query heads of the row share each staged key/value tile
// (the MQA reuse).  H = 64: each warp owns 16 heads and all 64 keys of a tile.
// H = 16: each warp owns the 16 heads and a quarter of the tile's keys; the
// four partial softmax states are merged at the end.  QK^T and PV run on bf16
// tensor-core MMAs with fp32 accumulation and an online (running max) softmax
// in the exp2 domain.  FP8 codes are widened to bf16 exactly and the per-entry
// scale is applied to the logits (nope part) and to the probabilities (value
// side), so no rounding is added to the cache values.  Decode rows split their
// slots over several CTAs; a combine kernel merges the partial states by their
// log-sum-exp.
#include "common.cuh"
#include "host_util.h"

namespace csa {
namespace {

constexpr int kKeys = 64;      // keys per staged tile
constexpr int kKS = kDQK + 8;  // padded bf16 row stride of the K tile (400 B)
constexpr int kVS = kDV + 8;   // padded bf16 row stride of the V tile (272 B)
constexpr int kThreads = 128;
constexpr size_t kSmemK = sizeof(__nv_bfloat16) * kKeys * kKS;
constexpr size_t kSmemV = sizeof(__nv_bfloat16) * kKeys * kVS;
constexpr size_t kSmemBytes = kSmemK + kSmemV + kKeys * (4 + 4 + 8);

struct AttnParams {
  const __nv_bfloat16* q;  // [R, H, 192]
  int64_t Tq, q_pos0;
  int H;
  int layout;
  int64_t N;
  const __nv_bfloat16* ck;
  const __nv_bfloat16* cv;
  const uint8_t* cnope;
  const __nv_bfloat16* crope;
  const float* cscale;
  int stride;
  const int32_t* idx;  // CSA: [R, k]; HCA: null (dense)
  int k;
  const __nv_bfloat16* wk;
  const __nv_bfloat16* wv;
  int64_t wpos0, wrows;
  int wlen;
  float scale_log2;
  int nsplit, tps;  // splits per row, tiles per split
  __nv_bfloat16* out;
  float* lse;
  float* part_o;   // [R, nsplit, H, 128]
  float* part_ml;  // [R, nsplit, H, 2]
};

__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(uint2 c) {
  uint4 v;
  v.x = e4m3x2_to_bf16x2(static_cast<uint16_t>(c.x & 0xffffu));
  v.y = e4m3x2_to_bf16x2(static_cast<uint16_t>(c.x >> 16));
  v.z = e4m3x2_to_bf16x2(static_cast<uint16_t>(c.y & 0xffffu));
  v.w = e4m3x2_to_bf16x2(static_cast<uint16_t>(c.y >> 16));
  return v;
}

// Writes one head row's result: final (bf16 + LSE) or a split partial.
__device__ __forceinline__ void emit_pair(const AttnParams& p, int64_t row, int split, int h, int d, float o0,
                                          float o1, float m, float l) {
  if (p.nsplit == 1) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    *reinterpret_cast<uint32_t*>(p.out + (row * p.H + h) * kDV + d) = pack_bf16x2(o0 * inv, o1 * inv);
  } else {
    *reinterpret_cast<float2*>(p.part_o + ((row * p.nsplit + split) * p.H + h) * kDV + d) = make_float2(o0, o1);
  }
}
__device__ __forceinline__ void emit_ml(const AttnParams& p, int64_t row, int split, int h, float m, float l) {
  if (p.nsplit == 1) {
    if (p.lse) p.lse[row * p.H + h] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
  } else {
    *reinterpret_cast<float2*>(p.part_ml + ((row * p.nsplit + split) * p.H + h) * 2) = make_float2(m, l);
  }
}

template <int KG>
__global__ void __launch_bounds__(kThreads) attn_kernel(AttnParams p) {
  constexpr int HG = 4 / KG;       // head groups of 16
  constexpr int KPW = kKeys / KG;  // keys per warp per tile
  constexpr int NTS = KPW / 8;     // S n-tiles per warp
  constexpr int KSP = KPW / 16;    // PV k-steps per warp
  extern __shared__ __align__(16) uint8_t smem[];
  auto Ks = reinterpret_cast<__nv_bfloat16(*)[kKS]>(smem);
  auto Vs = reinterpret_cast<__nv_bfloat16(*)[kVS]>(smem + kSmemK);
  float* sc = reinterpret_cast<float*>(smem + kSmemK + kSmemV);
  int* stype = reinterpret_cast<int*>(sc + kKeys);
  int64_t* srow = reinterpret_cast<int64_t*>(stype + kKeys);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hg = warp % HG, kg = warp / HG;
  const int64_t row = blockIdx.x;
  const int split = blockIdx.y;
  const int64_t b = row / p.Tq;
  const int64_t t = p.q_pos0 + row % p.Tq;
  const bool dense = p.idx == nullptr;
  int64_t n_ent;
  if (dense) {
    n_ent = (t + 1) / p.stride;
    if (n_ent > p.N) n_ent = p.N;
  } else {
    n_ent = p.k;
  }
  const int64_t wlo = (t - p.wlen + 1) > 0 ? (t - p.wlen + 1) : 0;
  const int64_t n_win = p.wlen > 0 ? (t - wlo + 1) : 0;
  const int64_t n_slots = n_ent + n_win;
  const int64_t slot_begin = static_cast<int64_t>(split) * p.tps * kKeys;
  int64_t slot_end = slot_begin + static_cast<int64_t>(p.tps) * kKeys;
  if (slot_end > n_slots) slot_end = n_slots;

  // Q as A fragments: heads hg*16 + (lane>>2) (+8), dims kk*16 + (lane&3)*2 (+8).
  uint32_t qf[12][4];
  {
    const __nv_bfloat16* qr = p.q + (row * p.H + hg * 16 + (lane >> 2)) * kDQK + (lane & 3) * 2;
#pragma unroll
    for (int kk = 0; kk < 12; ++kk) {
      qf[kk][0] = *reinterpret_cast<const uint32_t*>(qr + kk * 16);
      qf[kk][1] = *reinterpret_cast<const uint32_t*>(qr + 8 * kDQK + kk * 16);
      qf[kk][2] = *reinterpret_cast<const uint32_t*>(qr + kk * 16 + 8);
      qf[kk][3] = *reinterpret_cast<const uint32_t*>(qr + 8 * kDQK + kk * 16 + 8);
    }
  }
  float o[16][4];
#pragma unroll
  for (int nd = 0; nd < 16; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const bool fp8 = p.layout == CSA_KV_SPLIT_FP8;

  for (int64_t slot0 = slot_begin; slot0 < slot_end; slot0 += kKeys) {
    if (tid < kKeys) {
      const int64_t s = slot0 + tid;
      int type = 0;
      int64_t r = 0;
      if (s < slot_end) {
        if (s < n_ent) {
          const int64_t i = dense ? s : static_cast<int64_t>(p.idx[row * p.k + s]);
          if (i >= 0 && i < p.N && (i + 1) * p.stride - 1 <= t) {
            type = 1;
            r = b * p.N + i;
          }
        } else {
          const int64_t pos = wlo + (s - n_ent);
          type = 2;
          r = b * p.wrows + (pos - p.wpos0);
        }
      }
      stype[tid] = type;
      srow[tid] = r;
    }
    __syncthreads();
    for (int piece = tid; piece < kKeys * 24; piece += kThreads) {
      const int key = piece / 24, ch = piece % 24;
      const int type = stype[key];
      const int64_t r = srow[key];
      __nv_bfloat16* dst = &Ks[key][ch * 8];
      if (type == 0) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      } else if (type == 2) {
        cp_async16(dst, p.wk + r * kDQK + ch * 8);
      } else if (!fp8) {
        cp_async16(dst, p.ck + r * kDQK + ch * 8);
      } else if (ch < 16) {
        const uint4 v = e4m3x8_to_bf16x8(__ldg(reinterpret_cast<const uint2*>(p.cnope + r * kDNope + ch * 8)));
        *reinterpret_cast<uint4*>(dst) = v;
        *reinterpret_cast<uint4*>(&Vs[key][ch * 8]) = v;
      } else {
        cp_async16(dst, p.crope + r * kDRope + (ch - 16) * 8);
      }
    }
    for (int piece = tid; piece < kKeys * 16; piece += kThreads) {
      const int key = piece / 16, ch = piece % 16;
      const int type = stype[key];
      const int64_t r = srow[key];
      __nv_bfloat16* dst = &Vs[key][ch * 8];
      if (type == 0) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      } else if (type == 2) {
        cp_async16(dst, p.wv ? p.wv + r * kDV + ch * 8 : p.wk + r * kDQK + ch * 8);
      } else if (!fp8) {
        cp_async16(dst, p.cv ? p.cv + r * kDV + ch * 8 : p.ck + r * kDQK + ch * 8);
      }
    }
    if (tid < kKeys) sc[tid] = (fp8 && stype[tid] == 1) ? __ldg(p.cscale + srow[tid]) : 1.f;
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    const int kb = kg * KPW;
    float s[NTS][4];
#pragma unroll
    for (int nt = 0; nt < NTS; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    // nope channels
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int np = 0; np < NTS / 2; ++np) {
        const int key = kb + np * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
        const int dim = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(b0, b1, b2, b3, &Ks[key][dim]);
        mma_bf16(s[2 * np], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
        mma_bf16(s[2 * np + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
      }
    }
    // per-entry FP8 scale on the nope part of the logit
#pragma unroll
    for (int nt = 0; nt < NTS; ++nt) {
      const int key = kb + nt * 8 + (lane & 3) * 2;
      const float c0 = sc[key], c1 = sc[key + 1];
      s[nt][0] *= c0;
      s[nt][1] *= c1;
      s[nt][2] *= c0;
      s[nt][3] *= c1;
    }
    // RoPE channels
#pragma unroll
    for (int kk = 8; kk < 12; ++kk) {
#pragma unroll
      for (int np = 0; np < NTS / 2; ++np) {
        const int key = kb + np * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
        const int dim = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(b0, b1, b2, b3, &Ks[key][dim]);
        mma_bf16(s[2 * np], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
        mma_bf16(s[2 * np + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
      }
    }
    // mask, scale to the exp2 domain, running max
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NTS; ++nt) {
      const int key = kb + nt * 8 + (lane & 3) * 2;
      const bool v0 = stype[key] != 0, v1 = stype[key + 1] != 0;
      s[nt][0] = v0 ? s[nt][0] * p.scale_log2 : -INFINITY;
      s[nt][1] = v1 ? s[nt][1] * p.scale_log2 : -INFINITY;
      s[nt][2] = v0 ? s[nt][2] * p.scale_log2 : -INFINITY;
      s[nt][3] = v1 ? s[nt][3] * p.scale_log2 : -INFINITY;
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0;
    const float base1 = mn1 == -INFINITY ? 0.f : mn1;
    const float corr0 = exp2f(m0 - base0), corr1 = exp2f(m1 - base1);
    float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < NTS; ++nt) {
      s[nt][0] = exp2f(s[nt][0] - base0);
      s[nt][1] = exp2f(s[nt][1] - base0);
      s[nt][2] = exp2f(s[nt][2] - base1);
      s[nt][3] = exp2f(s[nt][3] - base1);
      sum0 += s[nt][0] + s[nt][1];
      sum1 += s[nt][2] + s[nt][3];
    }
    l0 = l0 * corr0 + sum0;
    l1 = l1 * corr1 + sum1;
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      o[nd][0] *= corr0;
      o[nd][1] *= corr0;
      o[nd][2] *= corr1;
      o[nd][3] *= corr1;
    }
    // O += (P * scale) V
#pragma unroll
    for (int ks = 0; ks < KSP; ++ks) {
      const int ka = kb + ks * 16 + (lane & 3) * 2;
      const float ca0 = sc[ka], ca1 = sc[ka + 1], cb0 = sc[ka + 8], cb1 = sc[ka + 9];
      const uint32_t a0 = pack_bf16x2(s[2 * ks][0] * ca0, s[2 * ks][1] * ca1);
      const uint32_t a1 = pack_bf16x2(s[2 * ks][2] * ca0, s[2 * ks][3] * ca1);
      const uint32_t a2 = pack_bf16x2(s[2 * ks + 1][0] * cb0, s[2 * ks + 1][1] * cb1);
      const uint32_t a3 = pack_bf16x2(s[2 * ks + 1][2] * cb0, s[2 * ks + 1][3] * cb1);
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {
        const int key = kb + ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int dim = dp * 16 + ((lane >> 4) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3, &Vs[key][dim]);
        mma_bf16(o[2 * dp], a0, a1, a2, a3, b0, b1);
        mma_bf16(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();
  }

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const int h0 = hg * 16 + (lane >> 2), h1 = h0 + 8;
  if (KG == 1) {
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      const int d = nd * 8 + (lane & 3) * 2;
      emit_pair(p, row, split, h0, d, o[nd][0], o[nd][1], m0, l0);
      emit_pair(p, row, split, h1, d, o[nd][2], o[nd][3], m1, l1);
    }
    if ((lane & 3) == 0) {
      emit_ml(p, row, split, h0, m0, l0);
      emit_ml(p, row, split, h1, m1, l1);
    }
    return;
  }
  // KG == 4: merge the four key-quarter states of the 16 heads through shared memory.
  float* mo = reinterpret_cast<float*>(smem);          // [4][16][128]
  float* ml = mo + 4 * 16 * kDV;                       // [4][16][2]
#pragma unroll
  for (int nd = 0; nd < 16; ++nd) {
    const int d = nd * 8 + (lane & 3) * 2;
    mo[(kg * 16 + (lane >> 2)) * kDV + d] = o[nd][0];
    mo[(kg * 16 + (lane >> 2)) * kDV + d + 1] = o[nd][1];
    mo[(kg * 16 + (lane >> 2) + 8) * kDV + d] = o[nd][2];
    mo[(kg * 16 + (lane >> 2) + 8) * kDV + d + 1] = o[nd][3];
  }
  if ((lane & 3) == 0) {
    ml[(kg * 16 + (lane >> 2)) * 2] = m0;
    ml[(kg * 16 + (lane >> 2)) * 2 + 1] = l0;
    ml[(kg * 16 + (lane >> 2) + 8) * 2] = m1;
    ml[(kg * 16 + (lane >> 2) + 8) * 2 + 1] = l1;
  }
  __syncthreads();
  const int h = tid >> 3;            // 16 heads x 8 dim segments of 16
  const int d0 = (tid & 7) * 16;
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < 4; ++w) M = fmaxf(M, ml[(w * 16 + h) * 2]);
  const float base = M == -INFINITY ? 0.f : M;
  float wgt[4], L = 0.f;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    wgt[w] = exp2f(ml[(w * 16 + h) * 2] - base);
    L += wgt[w] * ml[(w * 16 + h) * 2 + 1];
  }
#pragma unroll
  for (int d = 0; d < 16; d += 2) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      a0 += wgt[w] * mo[(w * 16 + h) * kDV + d0 + d];
      a1 += wgt[w] * mo[(w * 16 + h) * kDV + d0 + d + 1];
    }
    emit_pair(p, row, split, h, d0 + d, a0, a1, M, L);
  }
  if ((tid & 7) == 0) emit_ml(p, row, split, h, M, L);
}

// Merges split partials: one warp per (row, head), 4 channels per lane.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ part_o,
                                                      const float* __restrict__ part_ml, int64_t R, int H,
                                                      int nsplit, __nv_bfloat16* __restrict__ out,
                                                      float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (gw >= R * H) return;
  const int64_t row = gw / H;
  const int h = static_cast<int>(gw % H);
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, part_ml[((row * nsplit + s) * H + h) * 2]);
  const float base = M == -INFINITY ? 0.f : M;
  float L = 0.f, a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const int64_t e = (row * nsplit + s) * H + h;
    const float w = exp2f(part_ml[e * 2] - base);
    L += w * part_ml[e * 2 + 1];
    const float4 v = *reinterpret_cast<const float4*>(part_o + e * kDV + lane * 4);
    a0 += w * v.x;
    a1 += w * v.y;
    a2 += w * v.z;
    a3 += w * v.w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint2 pk = make_uint2(pack_bf16x2(a0 * inv, a1 * inv), pack_bf16x2(a2 * inv, a3 * inv));
  *reinterpret_cast<uint2*>(out + (row * H + h) * kDV + lane * 4) = pk;
  if (lane == 0 && lse) lse[row * H + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct Plan {
  int nsplit, tps;
  size_t ws;
};

size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

Plan plan(int64_t R, int H, int64_t max_slots) {
  Plan pl;
  const int64_t tiles = max_slots > 0 ? (max_slots + kKeys - 1) / kKeys : 1;
  const int64_t target = 2LL * num_sms();
  int64_t ns = 1;
  if (R < target) {
    ns = (target + R - 1) / R;
    if (ns > tiles) ns = tiles;
  }
  const int64_t tps = (tiles + ns - 1) / ns;
  ns = (tiles + tps - 1) / tps;
  pl.nsplit = static_cast<int>(ns);
  pl.tps = static_cast<int>(tps);
  pl.ws = ns > 1 ? align_up(static_cast<size_t>(R) * ns * H * kDV * 4) + align_up(static_cast<size_t>(R) * ns * H * 8)
                 : 0;
  return pl;
}

csa_status check_cache(const char* name, const csa_kv_cache* c) {
  if (c == nullptr) return fail(CSA_ERR_INVALID_ARG, "%s: cache is NULL", name);
  if (c->reserved != 0) return fail(CSA_ERR_INVALID_ARG, "%s: cache->reserved must be 0", name);
  if (c->n_entries < 0 || c->n_entries >= (1LL << 31))
    return fail(CSA_ERR_INVALID_ARG, "%s: cache->n_entries out of range", name);
  if (c->layout == CSA_KV_BF16) {
    if (c->n_entries > 0) {
      if (!c->k || !aligned16(c->k)) return fail(CSA_ERR_INVALID_ARG, "%s: cache->k NULL or misaligned", name);
      if (c->v && !aligned16(c->v)) return fail(CSA_ERR_INVALID_ARG, "%s: cache->v misaligned", name);
    }
  } else if (c->layout == CSA_KV_SPLIT_FP8) {
    if (c->n_entries > 0) {
      if (!c->nope || !aligned16(c->nope) || !c->rope || !aligned16(c->rope) || !c->scale)
        return fail(CSA_ERR_INVALID_ARG, "%s: split cache planes NULL or misaligned", name);
    }
  } else {
    return fail(CSA_ERR_INVALID_ARG, "%s: unknown cache layout %d", name, c->layout);
  }
  return CSA_OK;
}

csa_status run(const char* name, const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0,
               const csa_kv_cache* cache, int32_t stride, const int32_t* idx, int32_t k, const csa_window* win,
               float scale, void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  clear_error();
  CSA_REQUIRE(B >= 0 && Tq >= 0, "%s: negative size", name);
  CSA_REQUIRE(H == 16 || H == 64, "%s: H must be 16 or 64 (got %d)", name, H);
  CSA_REQUIRE(stride >= 1, "%s: stride must be >= 1", name);
  CSA_REQUIRE(q_pos0 >= 0, "%s: q_pos0 must be >= 0", name);
  CSA_REQUIRE(scale == scale && scale > -3.0e38f && scale < 3.0e38f, "%s: scale must be finite", name);
  if (csa_status st = check_cache(name, cache); st != CSA_OK) return st;
  const int64_t R = B * Tq;
  if (R == 0) return CSA_OK;
  CSA_REQUIRE(R < (1LL << 31), "%s: too many query rows", name);
  CSA_REQUIRE_PTR(q);
  CSA_REQUIRE_PTR(out);
  CSA_REQUIRE(lse == nullptr || (reinterpret_cast<uintptr_t>(lse) & 3u) == 0, "%s: lse misaligned", name);
  if (idx) CSA_REQUIRE(k >= 1 && k <= 4096 && aligned16(idx), "%s: idx misaligned or k out of [1, 4096]", name);
  int wlen = 0;
  if (win) {
    CSA_REQUIRE(win->reserved == 0 && win->len >= 0, "%s: bad window descriptor", name);
    wlen = win->len;
  }
  if (wlen > 0) {
    CSA_REQUIRE(win->k && aligned16(win->k), "%s: win->k NULL or misaligned", name);
    CSA_REQUIRE(!win->v || aligned16(win->v), "%s: win->v misaligned", name);
    const int64_t lo = (q_pos0 - wlen + 1) > 0 ? (q_pos0 - wlen + 1) : 0;
    const int64_t hi = q_pos0 + Tq - 1;
    CSA_REQUIRE(win->pos0 >= 0 && win->pos0 <= lo && hi < win->pos0 + win->rows,
                "%s: window rows [%lld, %lld) do not cover positions [%lld, %lld]", name,
                static_cast<long long>(win->pos0), static_cast<long long>(win->pos0 + win->rows),
                static_cast<long long>(lo), static_cast<long long>(hi));
  }
  const int64_t N = cache->n_entries;
  const int64_t max_slots = (idx ? k : N) + wlen;
  const Plan pl = plan(R, H, max_slots);
  if (pl.ws > 0 && (workspace == nullptr || workspace_bytes < pl.ws))
    return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed (got %zu)", name, pl.ws, workspace_bytes);
  if (pl.ws > 0) CSA_REQUIRE(aligned16(workspace), "%s: workspace misaligned", name);

  AttnParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.Tq = Tq;
  p.q_pos0 = q_pos0;
  p.H = H;
  p.layout = cache->layout;
  p.N = N;
  p.ck = static_cast<const __nv_bfloat16*>(cache->k);
  p.cv = static_cast<const __nv_bfloat16*>(cache->v);
  p.cnope = cache->nope;
  p.crope = static_cast<const __nv_bfloat16*>(cache->rope);
  p.cscale = cache->scale;
  p.stride = stride;
  p.idx = idx;
  p.k = idx ? k : 0;
  p.wk = wlen > 0 ? static_cast<const __nv_bfloat16*>(win->k) : nullptr;
  p.wv = wlen > 0 ? static_cast<const __nv_bfloat16*>(win->v) : nullptr;
  p.wpos0 = wlen > 0 ? win->pos0 : 0;
  p.wrows = wlen > 0 ? win->rows : 0;
  p.wlen = wlen;
  p.scale_log2 = scale * kLog2e;
  p.nsplit = pl.nsplit;
  p.tps = pl.tps;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = nullptr;
  p.part_ml = nullptr;
  if (pl.nsplit > 1) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.part_o = reinterpret_cast<float*>(ws);
    p.part_ml = reinterpret_cast<float*>(ws + align_up(static_cast<size_t>(R) * pl.nsplit * H * kDV * 4));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dim3 grid(static_cast<unsigned>(R), static_cast<unsigned>(pl.nsplit));
  prof_begin(s);
  if (H == 64)
    attn_kernel<1><<<grid, kThreads, kSmemBytes, s>>>(p);
  else
    attn_kernel<4><<<grid, kThreads, kSmemBytes, s>>>(p);
  prof_end(s);
  if (csa_status st = check_launch(name); st != CSA_OK) return st;
  if (pl.nsplit > 1) {
    const int64_t warps = R * H;
    combine_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, s>>>(p.part_o, p.part_ml, R, H, pl.nsplit,
                                                                           p.out, lse);
    return check_launch("attention combine");
  }
  return CSA_OK;
}

}  // namespace
}  // namespace csa

extern "C" {

size_t csa_sparse_mqa_workspace_size(int64_t B, int64_t Tq, int32_t H, int32_t k, int32_t win_len) {
  if (B <= 0 || Tq <= 0 || (H != 16 && H != 64) || k < 1 || win_len < 0) return 0;
  return csa::plan(B * Tq, H, static_cast<int64_t>(k) + win_len).ws;
}

size_t hca_dense_mqa_workspace_size(int64_t B, int64_t Tq, int32_t H, int64_t N, int32_t win_len) {
  if (B <= 0 || Tq <= 0 || (H != 16 && H != 64) || N < 0 || win_len < 0) return 0;
  return csa::plan(B * Tq, H, N + win_len).ws;
}

csa_status csa_sparse_mqa(const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0, const csa_kv_cache* cache,
                          int32_t m, const int32_t* idx, int32_t k, const csa_window* win, float scale, void* out,
                          float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (idx == nullptr && B * Tq > 0)
    return csa::fail(CSA_ERR_INVALID_ARG, "csa_sparse_mqa: idx is NULL");
  return csa::run("csa_sparse_mqa", q, B, Tq, H, q_pos0, cache, m, idx, k, win, scale, out, lse, workspace,
                  workspace_bytes, stream);
}

csa_status hca_dense_mqa(const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0, const csa_kv_cache* cache,
                         int32_t m_prime, const csa_window* win, float scale, void* out, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return csa::run("hca_dense_mqa", q, B, Tq, H, q_pos0, cache, m_prime, nullptr, 0, win, scale, out, lse, workspace,
                  workspace_bytes, stream);
}

}  // extern "C"
