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
// Each query row's key list is a sequence of "slots" (entry slots first, then
// window slots), processed in tiles of 64 keys.  A CTA of 4 warps owns one row
// and a contiguous range of its tiles; all query heads of the row share each
// staged key/value tile (the MQA reuse).  H = 64: each warp owns 16 heads and
// all keys of a tile; H = 16: each warp owns the 16 heads and a quarter of the
// tile's keys.  Tiles are double-buffered with cp.async: the next tile's rows
// (gathered by index for CSA, contiguous for HCA) stream in while the current
// one is multiplied.  FP8 codes are staged raw and widened to bf16 in shared
// memory (exact: every E4M3 value is a bf16 value); the per-entry scale is
// applied to the nope part of the logit and to the probability on the value
// side, so no rounding is added to cache values.  QK^T and PV are bf16
// tensor-core MMAs (fp32 accumulate) with an online softmax in the exp2 domain.
//
// Rows that are few (decode) split their tiles over a thread-block cluster of
// up to 16 CTAs; the partial softmax states (m, l, O) are merged through
// distributed shared memory inside the cluster, so there is no global
// scratch and no second launch.
#include <cooperative_groups.h>

#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "host_util.h"

namespace cg = cooperative_groups;

namespace csa {
namespace {

constexpr int kKeys = 64;      // keys per staged tile
constexpr int kKS = kDQK + 8;  // padded bf16 row stride of the K tile (400 B)
constexpr int kVS = kDV + 8;   // padded bf16 row stride of the V tile (272 B)
constexpr int kThreads = 128;
constexpr int kMaxCluster = 16;

struct AttnParams {
  const __nv_bfloat16* q;  // [R, H, 192]
  int64_t Tq, q_pos0;
  int H;
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
  int cl, tps;  // CTAs per row (cluster size), tiles per CTA
  __nv_bfloat16* out;
  float* lse;
};

struct SmemLayout {
  size_t ks, vs, raw, sc, stype, srow, idx, total;
};

__host__ __device__ constexpr size_t al16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

__host__ __device__ inline SmemLayout smem_layout(bool fp8, bool shv, int tps) {
  SmemLayout L;
  size_t off = 0;
  L.ks = off; off = al16(off + 2 * kKeys * kKS * sizeof(__nv_bfloat16));
  L.vs = off; if (!shv) off = al16(off + 2 * kKeys * kVS * sizeof(__nv_bfloat16));
  L.raw = off; if (fp8) off = al16(off + 2 * kKeys * kDNope);
  L.sc = off; off = al16(off + 2 * kKeys * sizeof(float));
  L.stype = off; off = al16(off + 2 * kKeys * sizeof(int));
  L.srow = off; off = al16(off + 2 * kKeys * sizeof(int64_t));
  L.idx = off; off = al16(off + static_cast<size_t>(tps) * kKeys * sizeof(int32_t));
  // merge buffer: ceil(H/cl) owned heads x cl*KG partials x (128 + 2) floats; H*KG == 64, so at most
  // (64 + 16 * 4) records when cl does not divide H (cl <= 16)
  const size_t reduce = (64 + 64) * (kDV + 2) * sizeof(float);
  L.total = off > reduce ? off : reduce;
  return L;
}

__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(uint32_t lo, uint32_t hi) {
  uint4 v;
  v.x = e4m3x2_to_bf16x2(static_cast<uint16_t>(lo & 0xffffu));
  v.y = e4m3x2_to_bf16x2(static_cast<uint16_t>(lo >> 16));
  v.z = e4m3x2_to_bf16x2(static_cast<uint16_t>(hi & 0xffffu));
  v.w = e4m3x2_to_bf16x2(static_cast<uint16_t>(hi >> 16));
  return v;
}

__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}

template <int KG, bool FP8, bool SHV>
__global__ void __launch_bounds__(kThreads) attn_kernel(AttnParams p) {
  constexpr int HG = 4 / KG;       // head groups of 16
  constexpr int KPW = kKeys / KG;  // keys per warp per tile
  constexpr int NTS = KPW / 8;     // S n-tiles per warp
  constexpr int KSP = KPW / 16;    // PV k-steps per warp
  extern __shared__ __align__(128) uint8_t smem[];
  const SmemLayout L = smem_layout(FP8, SHV, p.tps);
  auto Ks = reinterpret_cast<__nv_bfloat16(*)[kKeys][kKS]>(smem + L.ks);
  auto Vs = reinterpret_cast<__nv_bfloat16(*)[kKeys][kVS]>(smem + L.vs);
  auto raw = reinterpret_cast<uint8_t(*)[kKeys][kDNope]>(smem + L.raw);
  auto sc = reinterpret_cast<float(*)[kKeys]>(smem + L.sc);
  auto stype = reinterpret_cast<int(*)[kKeys]>(smem + L.stype);
  auto srow = reinterpret_cast<int64_t(*)[kKeys]>(smem + L.srow);
  int32_t* idx_s = reinterpret_cast<int32_t*>(smem + L.idx);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hg = warp % HG, kg = warp / HG;
  const int64_t row = blockIdx.x / p.cl;
  const int split = static_cast<int>(blockIdx.x % p.cl);
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
  const int64_t s0 = static_cast<int64_t>(split) * p.tps * kKeys;
  int64_t s1 = s0 + static_cast<int64_t>(p.tps) * kKeys;
  if (s1 > n_slots) s1 = n_slots;
  const int ntiles = s1 > s0 ? static_cast<int>((s1 - s0 + kKeys - 1) / kKeys) : 0;

  if (!dense) {  // this CTA's slice of the row's selection
    const int64_t e1 = s1 < n_ent ? s1 : n_ent;
    for (int64_t j = tid; j < e1 - s0; j += kThreads) idx_s[j] = p.idx[row * p.k + s0 + j];
  }

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

  // slot -> (type, source row): 0 skip, 1 compressed entry, 2 raw window token
  auto describe = [&](int tile, int st) {
    const int64_t s = s0 + static_cast<int64_t>(tile) * kKeys + tid;
    int type = 0;
    int64_t r = 0;
    if (s < s1) {
      if (s < n_ent) {
        const int64_t i = dense ? s : static_cast<int64_t>(idx_s[s - s0]);
        if (i >= 0 && i < p.N && (i + 1) * p.stride - 1 <= t) {
          type = 1;
          r = b * p.N + i;
        }
      } else {
        type = 2;
        r = b * p.wrows + (wlo + (s - n_ent) - p.wpos0);
      }
    }
    stype[st][tid] = type;
    srow[st][tid] = r;
  };
  auto issue = [&](int st) {
    for (int piece = tid; piece < kKeys * 24; piece += kThreads) {
      const int key = piece / 24, ch = piece % 24;
      const int type = stype[st][key];
      const int64_t r = srow[st][key];
      void* dst = &Ks[st][key][ch * 8];
      const void* src = p.q;
      int bytes = 16;
      if (type == 0) {
        bytes = 0;
      } else if (type == 2) {
        src = p.wk + r * kDQK + ch * 8;
      } else if (!FP8) {
        src = p.ck + r * kDQK + ch * 8;
      } else if (ch < 16) {
        if (ch & 1) continue;  // 8 chunks of 16 codes
        src = p.cnope + r * kDNope + (ch >> 1) * 16;
        dst = &raw[st][key][(ch >> 1) * 16];
      } else {
        src = p.crope + r * kDRope + (ch - 16) * 8;
      }
      cp_async16(dst, src, bytes);
    }
    if (!SHV) {
      for (int piece = tid; piece < kKeys * 16; piece += kThreads) {
        const int key = piece / 16, ch = piece % 16;
        const int type = stype[st][key];
        const int64_t r = srow[st][key];
        const void* src = p.q;
        int bytes = 16;
        if (type == 0 || (FP8 && type == 1)) {
          bytes = 0;  // FP8 entries get V from the widened codes
        } else if (type == 2) {
          src = p.wv ? p.wv + r * kDV + ch * 8 : p.wk + r * kDQK + ch * 8;
        } else {
          src = p.cv ? p.cv + r * kDV + ch * 8 : p.ck + r * kDQK + ch * 8;
        }
        cp_async16(&Vs[st][key][ch * 8], src, bytes);
      }
    }
    if (FP8 && tid < kKeys) {
      if (stype[st][tid] == 1)
        cp_async4(&sc[st][tid], p.cscale + srow[st][tid]);
      else
        sc[st][tid] = 1.f;
    }
  };
  auto widen = [&](int st) {  // FP8 codes -> bf16 nope channels (and V when not shared)
    for (int piece = tid; piece < kKeys * 8; piece += kThreads) {
      const int key = piece >> 3, c = piece & 7;
      if (stype[st][key] != 1) continue;
      const uint4 codes = *reinterpret_cast<const uint4*>(&raw[st][key][c * 16]);
      const uint4 lo = e4m3x8_to_bf16x8(codes.x, codes.y);
      const uint4 hi = e4m3x8_to_bf16x8(codes.z, codes.w);
      *reinterpret_cast<uint4*>(&Ks[st][key][c * 16]) = lo;
      *reinterpret_cast<uint4*>(&Ks[st][key][c * 16 + 8]) = hi;
      if (!SHV) {
        *reinterpret_cast<uint4*>(&Vs[st][key][c * 16]) = lo;
        *reinterpret_cast<uint4*>(&Vs[st][key][c * 16 + 8]) = hi;
      }
    }
  };

  if (ntiles > 0) {
    __syncthreads();  // idx_s
    if (tid < kKeys) describe(0, 0);
    __syncthreads();
    issue(0);
    cp_async_commit();
    if (ntiles > 1 && tid < kKeys) describe(1, 1);
    __syncthreads();
  }
  for (int tile = 0; tile < ntiles; ++tile) {
    const int st = tile & 1;
    if (tile + 1 < ntiles) issue(st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (FP8) {
      widen(st);
      __syncthreads();
    }
    const int kb = kg * KPW;
    float s[NTS][4];
#pragma unroll
    for (int nt = 0; nt < NTS; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 12; ++kk) {
      if (FP8 && kk == 8) {  // per-entry scale on the nope part of the logit
#pragma unroll
        for (int nt = 0; nt < NTS; ++nt) {
          const int key = kb + nt * 8 + (lane & 3) * 2;
          const float c0 = sc[st][key], c1 = sc[st][key + 1];
          s[nt][0] *= c0;
          s[nt][1] *= c1;
          s[nt][2] *= c0;
          s[nt][3] *= c1;
        }
      }
#pragma unroll
      for (int np = 0; np < NTS / 2; ++np) {
        const int key = kb + np * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
        const int dim = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(b0, b1, b2, b3, &Ks[st][key][dim]);
        mma_bf16(s[2 * np], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
        mma_bf16(s[2 * np + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
      }
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NTS; ++nt) {
      const int key = kb + nt * 8 + (lane & 3) * 2;
      const bool v0 = stype[st][key] != 0, v1 = stype[st][key + 1] != 0;
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
    const __nv_bfloat16* vbase = SHV ? &Ks[st][0][0] : &Vs[st][0][0];
    constexpr int vstride = SHV ? kKS : kVS;
#pragma unroll
    for (int ks = 0; ks < KSP; ++ks) {
      const int ka = kb + ks * 16 + (lane & 3) * 2;
      float ca0 = 1.f, ca1 = 1.f, cb0 = 1.f, cb1 = 1.f;
      if (FP8) {
        ca0 = sc[st][ka];
        ca1 = sc[st][ka + 1];
        cb0 = sc[st][ka + 8];
        cb1 = sc[st][ka + 9];
      }
      const uint32_t a0 = pack_bf16x2(s[2 * ks][0] * ca0, s[2 * ks][1] * ca1);
      const uint32_t a1 = pack_bf16x2(s[2 * ks][2] * ca0, s[2 * ks][3] * ca1);
      const uint32_t a2 = pack_bf16x2(s[2 * ks + 1][0] * cb0, s[2 * ks + 1][1] * cb1);
      const uint32_t a3 = pack_bf16x2(s[2 * ks + 1][2] * cb0, s[2 * ks + 1][3] * cb1);
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {
        const int key = kb + ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int dim = dp * 16 + ((lane >> 4) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3, vbase + key * vstride + dim);
        mma_bf16(o[2 * dp], a0, a1, a2, a3, b0, b1);
        mma_bf16(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();
    if (tile + 2 < ntiles && tid < kKeys) describe(tile + 2, st);
    __syncthreads();
  }
  cp_async_wait<0>();

  // ---- merge partial states (KG per CTA, cl CTAs per row) ----
  // Every warp pushes its partial (m, l, O) of each of its heads into the
  // shared memory of the head's owner CTA (h % cl), slot split*KG + kg; after
  // one cluster barrier each owner reduces its heads from local memory.
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  cg::cluster_group cluster = cg::this_cluster();
  if (p.cl > 1)
    cluster.sync();  // every CTA of the row is done with its tiles (the buffer reuses them)
  else
    __syncthreads();
  const int slots = p.cl * KG;
  float* rbuf = reinterpret_cast<float*>(smem);  // [heads owned][slots][kDV + 2]
  constexpr int kRec = kDV + 2;
  {
    const int slot = split * KG + kg;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int h = hg * 16 + (lane >> 2) + 8 * half;
      const int owner = h % p.cl;
      float* dst = (p.cl > 1 ? cluster.map_shared_rank(rbuf, owner) : rbuf) +
                   (static_cast<int64_t>(h / p.cl) * slots + slot) * kRec;
#pragma unroll
      for (int nd = 0; nd < 16; ++nd) {
        const int d = nd * 8 + (lane & 3) * 2;
        dst[d] = o[nd][2 * half];
        dst[d + 1] = o[nd][2 * half + 1];
      }
      if ((lane & 3) == 0) {
        dst[kDV] = half ? m1 : m0;
        dst[kDV + 1] = half ? l1 : l0;
      }
    }
  }
  if (p.cl > 1)
    cluster.sync();
  else
    __syncthreads();
  // this CTA owns heads h = split + j * cl; 32 threads x 4 channels per head
  const int sub = tid >> 5;
  for (int j = sub; split + j * p.cl < p.H; j += 4) {
    const int h = split + j * p.cl;
    const float* rec = rbuf + static_cast<int64_t>(j) * slots * kRec;
    float M = -INFINITY;
    for (int c = 0; c < slots; ++c) M = fmaxf(M, rec[c * kRec + kDV]);
    const float base = M == -INFINITY ? 0.f : M;
    float Lsum = 0.f, a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int c = 0; c < slots; ++c) {
      const float* r = rec + c * kRec;
      const float w = exp2f(r[kDV] - base);
      Lsum += w * r[kDV + 1];
      const float2 u = *reinterpret_cast<const float2*>(r + lane * 4);
      const float2 v = *reinterpret_cast<const float2*>(r + lane * 4 + 2);
      a0 += w * u.x;
      a1 += w * u.y;
      a2 += w * v.x;
      a3 += w * v.y;
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    *reinterpret_cast<uint2*>(p.out + (row * p.H + h) * kDV + lane * 4) =
        make_uint2(pack_bf16x2(a0 * inv, a1 * inv), pack_bf16x2(a2 * inv, a3 * inv));
    if (lane == 0 && p.lse) p.lse[row * p.H + h] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct Plan {
  int cl, tps;
};

Plan plan(int64_t R, int64_t max_slots) {
  const int64_t tiles = max_slots > 0 ? (max_slots + kKeys - 1) / kKeys : 1;
  const int64_t target = 2LL * num_sms();
  int64_t cl = 1;
  if (R < target) {
    cl = (target + R - 1) / R;
    if (cl > kMaxCluster) cl = kMaxCluster;
    if (cl > tiles) cl = tiles;
  }
  const int64_t tps = (tiles + cl - 1) / cl;
  cl = (tiles + tps - 1) / tps;
  return Plan{static_cast<int>(cl), static_cast<int>(tps)};
}

using KernelFn = void (*)(AttnParams);

KernelFn pick(int H, bool fp8, bool shv) {
  if (H == 64) {
    if (fp8) return shv ? attn_kernel<1, true, true> : attn_kernel<1, true, false>;
    return shv ? attn_kernel<1, false, true> : attn_kernel<1, false, false>;
  }
  if (fp8) return shv ? attn_kernel<4, true, true> : attn_kernel<4, true, false>;
  return shv ? attn_kernel<4, false, true> : attn_kernel<4, false, false>;
}

// Largest cluster size <= want that the device can co-schedule for this kernel.
int feasible_cluster(KernelFn fn, int want, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, int, size_t>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(dev, reinterpret_cast<const void*>(fn), want, smem);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int cl = want;
  while (cl > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cl));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = cl;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) == cudaSuccess && n > 0) break;
    cudaGetLastError();
    --cl;
  }
  cache[key] = cl;
  return cl;
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
      if (!c->nope || !aligned16(c->nope) || !c->rope || !aligned16(c->rope) || !c->scale ||
          (reinterpret_cast<uintptr_t>(c->scale) & 3u))
        return fail(CSA_ERR_INVALID_ARG, "%s: split cache planes NULL or misaligned", name);
    }
  } else {
    return fail(CSA_ERR_INVALID_ARG, "%s: unknown cache layout %d", name, c->layout);
  }
  return CSA_OK;
}

csa_status run(const char* name, const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0,
               const csa_kv_cache* cache, int32_t stride, const int32_t* idx, int32_t k, const csa_window* win,
               float scale, void* out, float* lse, void* stream) {
  clear_error();
  CSA_REQUIRE(B >= 0 && Tq >= 0, "%s: negative size", name);
  CSA_REQUIRE(H == 16 || H == 64, "%s: H must be 16 or 64 (got %d)", name, H);
  CSA_REQUIRE(stride >= 1, "%s: stride must be >= 1", name);
  CSA_REQUIRE(q_pos0 >= 0, "%s: q_pos0 must be >= 0", name);
  CSA_REQUIRE(scale == scale && scale > -3.0e38f && scale < 3.0e38f, "%s: scale must be finite", name);
  if (csa_status st = check_cache(name, cache); st != CSA_OK) return st;
  const int64_t R = B * Tq;
  if (R == 0) return CSA_OK;
  CSA_REQUIRE(R < (1LL << 31) / kMaxCluster, "%s: too many query rows", name);
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
  const bool fp8 = cache->layout == CSA_KV_SPLIT_FP8;
  const bool cache_shared_v = fp8 || cache->v == nullptr;
  const bool win_shared_v = wlen == 0 || win->v == nullptr;
  const bool shv = cache_shared_v && win_shared_v;
  const int64_t max_slots = (idx ? k : N) + wlen;
  Plan pl = plan(R, max_slots);
  KernelFn fn = pick(H, fp8, shv);
  size_t smem = smem_layout(fp8, shv, pl.tps).total;
  if (!ensure_smem(reinterpret_cast<const void*>(fn), static_cast<int>(smem)))
    return fail(CSA_ERR_CUDA, "%s: cannot raise the shared memory limit to %zu", name, smem);
  if (pl.cl > 1) {
    static std::mutex mu;
    {
      std::lock_guard<std::mutex> lock(mu);
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        pl.cl = pl.cl > 8 ? 8 : pl.cl;  // portable cluster sizes only
      }
    }
    const int cl = feasible_cluster(fn, pl.cl, smem);
    if (cl != pl.cl) {  // re-plan with the co-schedulable cluster size
      const int64_t tiles = max_slots > 0 ? (max_slots + kKeys - 1) / kKeys : 1;
      pl.tps = static_cast<int>((tiles + cl - 1) / cl);
      pl.cl = static_cast<int>((tiles + pl.tps - 1) / pl.tps);
      smem = smem_layout(fp8, shv, pl.tps).total;
      if (!ensure_smem(reinterpret_cast<const void*>(fn), static_cast<int>(smem)))
        return fail(CSA_ERR_CUDA, "%s: cannot raise the shared memory limit to %zu", name, smem);
    }
  }

  AttnParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.Tq = Tq;
  p.q_pos0 = q_pos0;
  p.H = H;
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
  p.cl = pl.cl;
  p.tps = pl.tps;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(R * pl.cl));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = pl.cl;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  prof_begin(cfg.stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fn, p);
  prof_end(cfg.stream);
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: launch failed: %s", name, cudaGetErrorString(e));
  return check_launch(name);
}

}  // namespace
}  // namespace csa

extern "C" {

size_t csa_sparse_mqa_workspace_size(int64_t B, int64_t Tq, int32_t H, int32_t k, int32_t win_len) {
  (void)B, (void)Tq, (void)H, (void)k, (void)win_len;
  return 0;  // partial states are merged in distributed shared memory
}

size_t hca_dense_mqa_workspace_size(int64_t B, int64_t Tq, int32_t H, int64_t N, int32_t win_len) {
  (void)B, (void)Tq, (void)H, (void)N, (void)win_len;
  return 0;
}

csa_status csa_sparse_mqa(const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0, const csa_kv_cache* cache,
                          int32_t m, const int32_t* idx, int32_t k, const csa_window* win, float scale, void* out,
                          float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  (void)workspace, (void)workspace_bytes;
  if (idx == nullptr && B * Tq > 0)
    return csa::fail(CSA_ERR_INVALID_ARG, "csa_sparse_mqa: idx is NULL");
  return csa::run("csa_sparse_mqa", q, B, Tq, H, q_pos0, cache, m, idx, k, win, scale, out, lse, stream);
}

csa_status hca_dense_mqa(const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0, const csa_kv_cache* cache,
                         int32_t m_prime, const csa_window* win, float scale, void* out, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream) {
  (void)workspace, (void)workspace_bytes;
  return csa::run("hca_dense_mqa", q, B, Tq, H, q_pos0, cache, m_prime, nullptr, 0, win, scale, out, lse, stream);
}

}  // extern "C"
