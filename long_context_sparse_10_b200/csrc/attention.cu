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
// window slots).  Three kernels cover the shapes:
//  - attn_tc_kernel (64 heads): one row per CTA (or a contiguous range of its
//    128-key tiles, for few rows), tcgen05 MMAs with the keys as the M
//    dimension; described where it is defined.
//  - attn_qblock_kernel (prefill over a bf16 cache: dense HCA attention, and
//    sparse CSA attention with few heads): blocks of consecutive queries,
//    256 (query, head) rows sharing each 64-key tile of the block's keys; dense
//    blocks on a persistent grid whose pipeline runs from block to block.
//  - attn_kernel (warp-level mma.sync, the remaining shapes: 16 heads with few
//    rows, an FP8 cache or packed sequences; 64 heads over an FP8 cache with a
//    separate raw-window V): one row per CTA in tiles of 64 keys,
//    double-buffered with cp.async; FP8 codes are widened in shared
//    memory and the per-entry scale applied to the nope part of the logit and
//    to the probability on the value side.
// All keep fp32 accumulators and an online softmax in the exp2 domain.
//
// Rows that are few (decode) split their tiles over several CTAs, merged in
// one of two ways: a thread-block cluster of up to 16 CTAs whose partial
// softmax states (m, l, O) meet in distributed shared memory (no global
// scratch, no second launch), or, on the tcgen05 path unless a cluster leaves
// no more tiles per CTA, one CTA per split writing 16-byte partial records to
// the caller's workspace, combined by attn_merge_kernel.
#include <cooperative_groups.h>

#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "host_util.h"
#include "tc.cuh"

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
  int cl, tps;  // CTAs per row (the splits of its slots), tiles per CTA
  __nv_bfloat16* out;
  float* lse;
  // Split records in global memory (tcgen05 path with several CTAs per row):
  // [R][cl][H][kRec] floats = unnormalised O (128), running max m (log2
  // units), sum l; merged by attn_merge_kernel.  Null: the CTAs of a row form
  // a thread-block cluster and merge through distributed shared memory.
  float* part;
  // Packed sequences (nullable): query row r belongs to the sequence s that
  // owns packed token r (cu_tok); its position is r - cu_tok[s], its entries
  // are cache rows [cu_ent[s], cu_ent[s+1]) and its window tokens are rows
  // cu_tok[s] + position of the raw-token buffer.
  const int32_t* cu_tok;
  const int32_t* cu_ent;
  int n_seqs;
  // rows of the cache planes and of the raw-token buffer (bounds of the
  // gathers, checked in builds with CSA_CHECKED)
  int64_t ent_rows, win_rows;
  int64_t qb_blocks;  // query-blocked kernel: B * ceil(Tq / (256 / H)) blocks
};

#ifdef CSA_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

// Where one query row's keys live: its position t, the cache row of its entry
// 0 (ebase) and its entry count N, and the raw-buffer row of position 0 (wbase).
struct RowGeo {
  int64_t t, ebase, N, wbase;
};
__device__ __forceinline__ RowGeo row_geo(const AttnParams& p, int64_t row) {
  RowGeo g;
  if (p.cu_tok != nullptr) {
    const int s = seq_of(p.cu_tok, p.n_seqs, row);
    const int64_t t0 = __ldg(p.cu_tok + s);
    g.t = row - t0;
    g.ebase = __ldg(p.cu_ent + s);
    g.N = __ldg(p.cu_ent + s + 1) - g.ebase;
    g.wbase = t0;
  } else {
    const int64_t b = row / p.Tq;
    g.t = p.q_pos0 + row % p.Tq;
    g.ebase = b * p.N;
    g.N = p.N;
    g.wbase = b * p.wrows - p.wpos0;
  }
  return g;
}

constexpr int kRec = kDV + 4;  // 128 channels, m, l, pad: 16-byte aligned records

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
  pdl_wait();
  pdl_trigger();
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
  const RowGeo geo = row_geo(p, row);
  const int64_t t = geo.t;
  const bool dense = p.idx == nullptr;
  int64_t n_ent;
  if (dense) {
    n_ent = (t + 1) / p.stride;
    if (n_ent > geo.N) n_ent = geo.N;
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
        if (i >= 0 && i < geo.N && (i + 1) * p.stride - 1 <= t) {
          type = 1;
          r = geo.ebase + i;
        }
      } else {
        type = 2;
        r = geo.wbase + (wlo + (s - n_ent));
      }
    }
    if (type != 0 && !CSA_INBOUNDS(r >= 0 && r < (type == 1 ? p.ent_rows : p.win_rows))) type = 0;
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
// H = 64: tcgen05 path, with the keys as the MMA's M dimension.  One query's
// 64 heads share every key (MQA), so instead of S = Q K^T (M = 64 heads, a
// half-rate shape) the tensor cores compute
//   S^T = K Q^T     M = 128 keys,     N = 64 heads, K = 192 dims  (12 MMAs)
//   O^T += V^T P^T  M = 128 channels, N = 64 heads, K = 128 keys  (8 MMAs)
//   l^T += 1 P^T    M = 128 (all rows equal), N = 64 heads        (8 MMAs)
// all at M = 128, with fp32 accumulators in tensor memory: S^T double-buffered
// in columns [0, 128), O^T in [128, 192), the running sums l in [192, 256).
// Softmax warps 0-7: thread (warp w, lane l) owns TMEM lane 32 (w % 4) + l,
// i.e. that key of the tile, and heads 32 (w / 4) .. +31: it reads those
// logits and writes its half of the key's P^T row (the row is 128 bytes, the
// B operand's MN-major layout) to shared memory.  The running max per head
// (m_ref, shared memory) changes only when some logit exceeds it by more
// than 2^20 (log2 units) -- always on a CTA's first tile, rarely after; then
// the tile's per-head maxima are reduced across the 128 keys (a halving
// shuffle per warp), O and l are rescaled in TMEM, and the tile continues.
// Operands sit in shared memory in the 128-byte-swizzled layout: K K-major
// (three 64-dim blocks), Q K-major, V^T read MN-major straight out of the
// first two K blocks when key and value are shared, P^T MN-major, and the
// all-ones A operand of the l update is one 1 KB swizzle atom read with a
// zero row-group stride.  Warps 8-15 gather key tiles: FP8 entries are
// dequantised (code x scale rounded to bf16, from registers into the K tile);
// bf16 rows are copied with cp.async whose completions arrive on the stage
// barrier themselves, K stages released when S is done and V stages when PV
// is (separate V).  One thread of warp 16 issues every MMA: S(0), S(1), then
// whichever is ready first of PV(t) + the l update (once P(t) is written) and
// S(t+2) (once its keys are in and PV(t) has gone out, so that S(t+2)'s
// commit also releases P buffer t % 2).  When key and value are shared the K
// tile has three stages (two with a separate V tile).  Every mbarrier wait is
// bounded; a timeout sets the device error word instead of hanging.
// ---------------------------------------------------------------------------
constexpr int kTcKeys = 128;

constexpr int kTcDecThreads = 544;  // attn_tc_kernel: warps 0-7 softmax, 8-15 loads, 16 MMA issue
constexpr float kRescaleLog2 = 20.f;  // rescale O and l when a logit tops m_ref by more than 2^20
// The first tile of a CTA tries the reference 0 for every head: kept when
// every head has a valid logit of at least kFloorLog2 (so that the largest
// probabilities are far from the fp32 / bf16 underflow) and none above
// kRescaleLog2; otherwise the exact per-head maxima are reduced.
constexpr float kFloorLog2 = -64.f;

struct TcLayout {
  size_t q, k, v, p, ones, stype, srow, mref, corr, wmax, hseen, bars, total;
};

// Slot types of the last four tiles (ring indexed by tile % 4): 0 skipped, 1
// compressed entry, 2 raw window token.  A tile's slot is rewritten only after
// the softmax of the tile four back has finished with it.
constexpr int kTypeRing = 4;


// K-tile stages: three when the V tile is the K tile, two otherwise.
__host__ __device__ constexpr int tc_stages(bool fp8, bool shv) { return (void)fp8, shv ? 3 : 2; }

__host__ __device__ inline TcLayout tc_layout(bool fp8, bool shv, int tps) {
  TcLayout L;
  const int ns = tc_stages(fp8, shv);
  size_t off = 0;
  L.q = off; off += 3 * 8192;                    // Q: 64 heads x 192 dims
  L.k = off; off += ns * 3 * 16384;              // K: stages x 128 keys x 192 dims
  L.v = off; if (!shv) off += ns * 2 * 16384;    // V: stages x 128 keys x 128 dims
  L.p = off; off += 2 * 16384;                   // P^T: 2 buffers x 128 keys x 64 heads (epilogue: O^T transpose)
  L.ones = off; off += 1024;                     // all-ones swizzle atom
  L.stype = off; off += kTypeRing * kTcKeys * sizeof(int);
  L.srow = off; off += kTypeRing * kTcKeys * sizeof(int64_t);
  L.mref = off; off += 64 * sizeof(float);
  L.corr = off; off += 64 * sizeof(float);
  L.wmax = off; off += 4 * 64 * sizeof(float);
  L.hseen = off; off += 16;                      // 64 head flags of the first tile's trial reference
  L.bars = off; off += 128;
  (void)fp8, (void)tps;
  const size_t reduce = 80 * (kDV + 4) * sizeof(float);  // cluster merge records (reuse Q/K)
  L.total = (off > reduce ? off : reduce) + 1024;          // + alignment slack
  return L;
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
// Named barrier that also ORs a predicate over the participating threads.
__device__ __forceinline__ bool named_sync_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n.reg .pred pi, po;\nsetp.ne.u32 pi, %1, 0;\nbarrier.red.or.pred po, %2, %3, pi;\nselp.u32 %0, 1, 0, po;\n}\n"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
// Arrives on `bar` once every cp.async this thread has issued so far has
// landed (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

// Per-head maximum over the 32 lanes of a warp, each lane holding v[0..31]
// (one key, 32 heads): five halving exchange steps (31 shuffles); returns in
// v[0] the maximum of head bitrev-ordered h0 below.
__device__ __forceinline__ int warp_head_max32(float* v, int lane) {
#pragma unroll
  for (int w = 16, o = 16; o >= 1; w >>= 1, o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float keep = up ? v[i + w] : v[i];
      const float send = up ? v[i] : v[i + w];
      v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
    }
  }
  return ((lane >> 4) & 1) * 16 + ((lane >> 3) & 1) * 8 + ((lane >> 2) & 1) * 4 + ((lane >> 1) & 1) * 2 + (lane & 1);
}

// 2^x by the hardware approximation (relative error ~2^-22, far below the
// bf16 rounding of the probabilities it feeds); 0 for x = -inf.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <bool FP8, bool SHV>
__global__ void __launch_bounds__(kTcDecThreads, 1) attn_tc_kernel(AttnParams p) {
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const TcLayout L = tc_layout(FP8, SHV, p.tps);
  uint8_t* Qs = smem + L.q;
  uint8_t* Kst = smem + L.k;
  uint8_t* Vst = smem + L.v;
  uint8_t* Pst = smem + L.p;
  uint8_t* ones = smem + L.ones;
  constexpr int NS = tc_stages(FP8, SHV);
  auto stype = reinterpret_cast<int(*)[kTcKeys]>(smem + L.stype);  // [tile % kTypeRing][slot]
  auto srow = reinterpret_cast<int64_t(*)[kTcKeys]>(smem + L.srow);
  float* mref = reinterpret_cast<float*>(smem + L.mref);
  float* corr_s = reinterpret_cast<float*>(smem + L.corr);
  auto wmax = reinterpret_cast<float(*)[64]>(smem + L.wmax);
  uint32_t* hseen = reinterpret_cast<uint32_t*>(smem + L.hseen);  // [2]: heads 0-31, 32-63
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);  // [NS] K stage loaded
  uint64_t* empty = full + NS;                                    // [NS] PV of the stage's tile done
  uint64_t* sdone = empty + NS;                                   // [2] S of the tile done (TMEM buffer)
  uint64_t* pready = sdone + 2;                                   // [2] P of the tile written (smem buffer)
  uint64_t* vfull = pready + 2;                                   // [2] V stage loaded (bf16, separate V)
  uint64_t* kfree = vfull + 2;                                    // [2] S of the K stage's tile done (same)
  uint32_t* tslot = reinterpret_cast<uint32_t*>(kfree + 2);
  // bf16 cache with a separate V: K stages are released when S is done, V
  // stages when PV is, so the next K tiles stream in while P and PV run
  constexpr bool kSplitKV = !FP8 && !SHV;
  constexpr int kKB = 16384;  // one 64-dim block of a 128-key tile

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t row = blockIdx.x / p.cl;
  const int split = static_cast<int>(blockIdx.x % p.cl);
  const RowGeo geo = row_geo(p, row);
  const int64_t t = geo.t;
  const bool dense = p.idx == nullptr;
  int64_t n_ent;
  if (dense) {
    n_ent = (t + 1) / p.stride;
    if (n_ent > geo.N) n_ent = geo.N;
  } else {
    n_ent = p.k;
  }
  const int64_t wlo = (t - p.wlen + 1) > 0 ? (t - p.wlen + 1) : 0;
  const int64_t n_win = p.wlen > 0 ? (t - wlo + 1) : 0;
  const int64_t n_slots = n_ent + n_win;
  const int64_t s0 = static_cast<int64_t>(split) * p.tps * kTcKeys;
  int64_t s1 = s0 + static_cast<int64_t>(p.tps) * kTcKeys;
  if (s1 > n_slots) s1 = n_slots;
  const int ntiles = s1 > s0 ? static_cast<int>((s1 - s0 + kTcKeys - 1) / kTcKeys) : 0;

  if (tid == 0) {
    // bf16 path: a loaded stage counts one arrival per producer thread, made
    // by its copies (see the producer); the FP8 producer arrives once
    for (int i = 0; i < 2 * NS + 8; ++i) {
      const bool loaded = i < NS || (i >= 2 * NS + 4 && i < 2 * NS + 6);  // full[], vfull[]
      tc::bar_init(&full[i], (!FP8 && loaded) ? 256 : 1);
    }
    tc::bar_init_fence();
  }
  __syncthreads();  // the barriers exist
  // FP8 cache (decode: a few tiles per CTA): the consumers (softmax warps 0-7
  // and the MMA warp 16) set up TMEM, Q and the running maxima while the
  // producer gathers the first tiles.  bf16 cache (long prefill rows): every
  // thread loads Q first (measured faster there).
  const bool consumer = !FP8 || warp < 8 || warp == 16;
  if (consumer) {
    const int nct = FP8 ? 288 : kTcDecThreads;
    const int ct = !FP8 ? tid : (warp < 8 ? tid : 256 + lane);
    if (warp == 0) tc::tmem_alloc(tslot, 256);
    for (int piece = ct; piece < 64 * 24; piece += nct) {  // Q, swizzled K-major
      const int hh = piece / 24, ch = piece % 24;
      cp_async16(Qs + (ch >> 3) * 8192 + tc::sw128(hh, ch & 7), p.q + (row * 64 + hh) * kDQK + ch * 8);
    }
    cp_async_commit();
    if (tid < 64) {
      reinterpret_cast<uint4*>(ones)[tid] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
      mref[tid] = -INFINITY;
      if (tid < 2) hseen[tid] = 0u;
    }
    cp_async_wait<0>();
    tc::fence_async_smem();
    tc::fence_before_sync();
    named_sync(5, nct);
    tc::fence_after_sync();
  }
  const uint32_t tmem = consumer ? *tslot : 0u;
  bool healthy = true;  // false after a barrier wait ran out: later waits are skipped
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t tO = tmem + 128, tL = tmem + 192;

  constexpr uint32_t kIdescS = tc::idesc_bf16(128, 64, false, false);  // A = K (K-major), B = Q (K-major)
  constexpr uint32_t kIdescO = tc::idesc_bf16(128, 64, true, true);    // A = V^T (MN-major), B = P^T (MN-major)
  constexpr uint32_t kIdescL = tc::idesc_bf16(128, 64, true, false);   // A = ones, B = P^T (MN-major)
  if (warp == 16) {
    // ===================== MMA issue (one thread) =====================
    // A commit tracks every earlier MMA of this thread: S(t+2) done implies
    // PV(t) done, which frees P buffer t % 2 for tile t+2.
    auto issue_s = [&](int tile) {
      const int kst = tile % NS;
      const uint32_t tS = tmem + 64 * (tile & 1);
      const uint32_t qa = smem_u32(Qs), ka = smem_u32(Kst + kst * 3 * kKB);
      if (!FP8) tc::fence_async_smem();  // the stage was written by cp.async
      tc::fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < 12; ++kk) {
        const uint64_t adesc = tc::desc_sw128(ka + (kk >> 2) * kKB + (kk & 3) * 32, 16, 1024);
        const uint64_t bdesc = tc::desc_sw128(qa + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
        tc::mma_bf16_ss(tS, adesc, bdesc, kIdescS, kk > 0 ? 1u : 0u);
      }
      tc::mma_commit(&sdone[tile & 1]);
      if (kSplitKV) tc::mma_commit(&kfree[kst]);
    };
    const uint64_t onesdesc = tc::desc_sw128(smem_u32(ones), 16, 0);
    auto issue_pv = [&](int tile) {
      const int kst = tile % NS, pb = tile & 1;
      if (!FP8) tc::fence_async_smem();  // the stage was written by cp.async
      tc::fence_after_sync();
      const uint32_t pa = smem_u32(Pst + pb * 16384);
      const uint32_t va = SHV ? smem_u32(Kst + kst * 3 * kKB) : smem_u32(Vst + kst * 2 * kKB);
#pragma unroll
      for (int ks = 0; ks < kTcKeys / 16; ++ks) {
        const uint64_t pdesc = tc::desc_sw128(pa + ks * 2048, 8192, 1024);
        const uint32_t acc = (tile > 0 || ks > 0) ? 1u : 0u;
        tc::mma_bf16_ss(tO, tc::desc_sw128(va + ks * 2048, kKB, 1024), pdesc, kIdescO, acc);
        tc::mma_bf16_ss(tL, onesdesc, pdesc, kIdescL, acc);
      }
      tc::mma_commit(&empty[kst]);
    };
    if (lane == 0 && ntiles > 0) {
      for (int t0 = 0; t0 < 2 && t0 < ntiles; ++t0) {
        if (healthy) healthy = tc::bar_wait(&full[t0 % NS], (t0 / NS) & 1);
        issue_s(t0);
      }
      // Whichever is ready first: PV(next_pv) once its P (and V) are in, or
      // S(next_s) once its K stage is loaded and PV(next_s - 2) has been issued
      // (S(next_s) reuses the TMEM buffer and, through its commit, releases
      // the P buffer of tile next_s - 2).  Neither waits behind the other.
      int next_pv = 0, next_s = 2;
      uint32_t idle = 0;
      while (next_pv < ntiles && healthy) {
        bool moved = false;
        if (next_s < ntiles && next_s - 2 < next_pv && tc::bar_test(&full[next_s % NS], (next_s / NS) & 1)) {
          issue_s(next_s);
          ++next_s;
          moved = true;
        }
        if (tc::bar_test(&pready[next_pv & 1], (next_pv >> 1) & 1) &&
            (!kSplitKV || tc::bar_test(&vfull[next_pv % NS], (next_pv / NS) & 1))) {
          issue_pv(next_pv);
          ++next_pv;
          moved = true;
        }
        if (moved) {
          idle = 0;
        } else if (++idle > tc::kPollLimit) {
          atomicExch(&tc::g_device_error, tc::kErrWaitTimeout);
          healthy = false;
        }
      }
    }
  } else if (warp >= 8) {
    if constexpr (!FP8) {
      // ===================== producer (bf16 cache): asynchronous gathers =====================
      // 256 threads copy each tile with 16-byte cp.async and let the copies
      // themselves arrive on the stage barrier (cp.async.mbarrier.arrive.noinc,
      // 256 arrivals), so the producer never waits for its own data: it only
      // waits for a stage to be free.  K(t+1) is issued before V(t): K stages
      // are freed when S is done, V stages when PV is (separate V); with a
      // shared V the K stage is freed by PV.
      const int pt = tid - 256;  // 0..255; threads 0..127 also own one slot each
      const int pwarp = warp - 8;
      auto load_sel = [&](int tile) -> int32_t {
        const int64_t sl = s0 + static_cast<int64_t>(tile) * kTcKeys + pt;
        return (!dense && pt < kTcKeys && tile < ntiles && sl < s1 && sl < n_ent) ? __ldg(p.idx + row * p.k + sl)
                                                                                  : -1;
      };
      // The tile's slots are an entry run [0, ne) then a window run [ne, ne + nw).
      auto runs = [&](int tile, int& ne, int& nw) {
        const int64_t a0 = s0 + static_cast<int64_t>(tile) * kTcKeys;
        const int64_t a1 = (a0 + kTcKeys) < s1 ? (a0 + kTcKeys) : s1;
        const int64_t e1 = a1 < n_ent ? a1 : n_ent;
        ne = static_cast<int>(e1 - a0 > 0 ? e1 - a0 : 0);
        nw = static_cast<int>(a1 - a0) - ne;
      };
      // nch 16-byte chunks per key from a source row of `stride` elements:
      // K = 24 chunks (three 64-dim blocks), V = 16 chunks (two blocks)
      auto issue = [&](uint8_t* T, int tile, int nch, const __nv_bfloat16* esrc, int estride,
                       const __nv_bfloat16* wsrc, int wstride) {
        const int ring = tile & (kTypeRing - 1);
        int ne, nw;
        runs(tile, ne, nw);
        if (ne > 0 && dense && !kChecked) {  // contiguous entry rows
          const int64_t r0 = srow[ring][0];
          for (int pc = pt; pc < ne * nch; pc += 256) {
            const int key = pc / nch, c = pc % nch;
            cp_async16(T + (c >> 3) * kKB + tc::sw128(key, c & 7), esrc + (r0 + key) * estride + c * 8);
          }
        } else if (ne > 0) {  // selected entries: four keys per warp instruction, 8 lanes per 128-byte row
          const int c = lane & 7;
          for (int kb = pwarp * 4; kb < ne; kb += 32) {
            const int key = kb + (lane >> 3);
            if (key >= ne) continue;
            const int type = stype[ring][key];
            const int64_t r = srow[ring][key];
            for (int j = 0; j < nch / 8; ++j)
              cp_async16(T + j * kKB + tc::sw128(key, c), type ? esrc + r * estride + (8 * j + c) * 8 : p.q,
                         type ? 16 : 0);
          }
        }
        if (nw > 0) {  // raw window tokens: contiguous rows
          const int64_t rw0 = srow[ring][ne];
          const bool inb = CSA_INBOUNDS(rw0 >= 0 && rw0 + nw <= p.win_rows);
          for (int pc = pt; pc < nw * nch; pc += 256) {
            const int key = ne + pc / nch, c = pc % nch;
            cp_async16(T + (c >> 3) * kKB + tc::sw128(key, c & 7),
                       inb ? wsrc + (rw0 + pc / nch) * wstride + c * 8 : p.q, inb ? 16 : 0);
          }
        }
        for (int pc = pt; pc < (kTcKeys - ne - nw) * nch; pc += 256) {  // past the row's end: zero rows
          const int key = ne + nw + pc / nch, c = pc % nch;
          cp_async16(T + (c >> 3) * kKB + tc::sw128(key, c & 7), p.q, 0);
        }
      };
      const __nv_bfloat16* ve = p.cv ? p.cv : p.ck;
      const int ves = p.cv ? kDV : kDQK;
      const __nv_bfloat16* vw = p.wv ? p.wv : p.wk;
      const int vws = p.wv ? kDV : kDQK;
      int32_t sel_next = load_sel(0);
      for (int it = 0; it <= ntiles; ++it) {
        if (it < ntiles) {  // K of tile `it`
          const int tile = it, st = tile % NS, ring = tile & (kTypeRing - 1);
          const int32_t sel_cur = sel_next;
          sel_next = load_sel(tile + 1);
          if (pt < kTcKeys) {  // slot -> (type, row): 0 skip, 1 compressed entry, 2 raw window token
            const int64_t sl = s0 + static_cast<int64_t>(tile) * kTcKeys + pt;
            int type = 0;
            int64_t r = 0;
            if (sl < s1) {
              if (sl < n_ent) {
                const int64_t i = dense ? sl : static_cast<int64_t>(sel_cur);
                if (i >= 0 && i < geo.N && (i + 1) * p.stride - 1 <= t) {
                  type = 1;
                  r = geo.ebase + i;
                }
              } else {
                type = 2;
                r = geo.wbase + (wlo + (sl - n_ent));
              }
            }
            if (type != 0 && !CSA_INBOUNDS(r >= 0 && r < (type == 1 ? p.ent_rows : p.win_rows))) type = 0;
            stype[ring][pt] = type;
            srow[ring][pt] = r;
          }
          bool ok = true;
          if (tile >= NS) ok = tc::bar_wait(kSplitKV ? &kfree[st] : &empty[st], ((tile / NS) - 1) & 1);
          if (named_sync_or(1, 256, !ok)) {  // also publishes the slot table to the 256 threads
            healthy = false;
            break;
          }
          issue(Kst + st * 3 * kKB, tile, 24, p.ck, kDQK, p.wk, kDQK);
          cp_async_mbar_arrive_noinc(&full[st]);
        }
        if (kSplitKV && it >= 1) {  // V of tile `it - 1`
          const int tile = it - 1, vs = tile % NS;
          bool ok = true;
          if (tile >= NS) ok = tc::bar_wait(&empty[vs], ((tile / NS) - 1) & 1);
          if (named_sync_or(3, 256, !ok)) {
            healthy = false;
            break;
          }
          issue(Vst + vs * 2 * kKB, tile, 16, ve, ves, vw, vws);
          cp_async_mbar_arrive_noinc(&vfull[vs]);
        }
      }
      cp_async_wait<0>();  // no copy of this thread is left in flight when the CTA moves on
    } else {
      // ===================== producer: gather, widen, publish =====================
      const int pt = tid - 256;  // 0..255; threads 0..127 also own one slot each
      // selected entry of this thread's slot in the next tile, loaded one tile
      // ahead so that its latency overlaps the current tile's gathers
      auto load_sel = [&](int tile) -> int32_t {
        const int64_t sl = s0 + static_cast<int64_t>(tile) * kTcKeys + pt;
        return (!dense && pt < kTcKeys && tile < ntiles && sl < s1 && sl < n_ent) ? __ldg(p.idx + row * p.k + sl) : -1;
      };
      int32_t sel_next = load_sel(0);
      for (int tile = 0; tile < ntiles; ++tile) {
        const int st = tile % NS;
        const int32_t sel_cur = sel_next;
        if (tile >= NS && healthy) healthy = tc::bar_wait(&empty[st], ((tile / NS) - 1) & 1);
        // slot -> (type, row): 0 skip, 1 compressed entry, 2 raw window token
        if (pt < kTcKeys) {
          const int64_t sl = s0 + static_cast<int64_t>(tile) * kTcKeys + pt;
          int type = 0;
          int64_t r = 0;
          if (sl < s1) {
            if (sl < n_ent) {
              const int64_t i = dense ? sl : static_cast<int64_t>(sel_cur);
              if (i >= 0 && i < geo.N && (i + 1) * p.stride - 1 <= t) {
                type = 1;
                r = geo.ebase + i;
              }
            } else {
              type = 2;
              r = geo.wbase + (wlo + (sl - n_ent));
            }
          }
          if (type != 0 && !CSA_INBOUNDS(r >= 0 && r < (type == 1 ? p.ent_rows : p.win_rows))) type = 0;
          stype[tile & (kTypeRing - 1)][pt] = type;
          srow[st][pt] = r;
        }
        named_sync(1, 256);
        uint8_t* Kt = Kst + st * 3 * kKB;
        uint8_t* Vt = Vst + st * 2 * kKB;
        // The tile's slots are an entry run [0, ne) then a window run [ne, ne + nw).
        const int64_t a0 = s0 + static_cast<int64_t>(tile) * kTcKeys;
        const int64_t a1 = (a0 + kTcKeys) < s1 ? (a0 + kTcKeys) : s1;
        const int ne = static_cast<int>(((a1 < n_ent ? a1 : n_ent) - a0) > 0 ? ((a1 < n_ent ? a1 : n_ent) - a0) : 0);
        const int nw = static_cast<int>(a1 - a0) - ne;
        const int pwarp = warp - 8;
        // FP8 entries: thread pt owns 16-code chunk c = pt % 8 of keys pt / 8 + 32 j
        // (eight lanes per 128-byte row, four rows per warp instruction); the
        // codes and scales go to registers here and are widened after the
        // asynchronous copies below are issued.
        uint4 codes[4];
        float scl[4];
        if (FP8) {
  #pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int key = (pt >> 3) + 32 * j;
            const bool ok = key < ne && stype[tile & (kTypeRing - 1)][key] == 1;
            const int64_t r = ok ? srow[st][key] : 0;
            codes[j] = ok ? ldg_nc16(p.cnope + r * kDNope + (pt & 7) * 16) : make_uint4(0u, 0u, 0u, 0u);
            scl[j] = ok ? __ldg(p.cscale + r) : 0.f;
          }
        }
        // Contiguous runs are copied with consecutive lanes on consecutive 16-byte
        // chunks (512-byte warp requests); selected entries are gathered four keys
        // per warp instruction (8 lanes per 128-byte row).
        if (ne > 0 && dense && !kChecked) {
          const int64_t r0 = srow[st][0];
          if (FP8) {
            for (int pc = pt; pc < ne * 8; pc += 256)
              cp_async16(Kt + 2 * kKB + tc::sw128(pc >> 3, pc & 7), p.crope + r0 * kDRope + pc * 8);
          } else {
            for (int pc = pt; pc < ne * 24; pc += 256) {
              const int key = pc / 24, c = pc % 24;
              cp_async16(Kt + (c >> 3) * kKB + tc::sw128(key, c & 7), p.ck + r0 * kDQK + pc * 8);
            }
            if (!SHV) {
              for (int pc = pt; pc < ne * 16; pc += 256) {
                const int key = pc >> 4, c = pc & 15;
                const __nv_bfloat16* src = p.cv ? p.cv + r0 * kDV + pc * 8 : p.ck + (r0 + key) * kDQK + c * 8;
                cp_async16(Vt + (c >> 3) * kKB + tc::sw128(key, c & 7), src);
              }
            }
          }
        } else if (ne > 0) {
          const int c = lane & 7;
          for (int kb = pwarp * 4; kb < ne; kb += 32) {
            const int key = kb + (lane >> 3);
            if (key >= ne) continue;
            const int type = stype[tile & (kTypeRing - 1)][key];
            const int64_t r = srow[st][key];
            const int bytes = type ? 16 : 0;
            if (FP8) {
              cp_async16(Kt + 2 * kKB + tc::sw128(key, c), type ? p.crope + r * kDRope + c * 8 : p.crope, bytes);
            } else {
  #pragma unroll
              for (int j = 0; j < 3; ++j)
                cp_async16(Kt + j * kKB + tc::sw128(key, c), type ? p.ck + r * kDQK + (8 * j + c) * 8 : p.ck, bytes);
              if (!SHV) {
  #pragma unroll
                for (int j = 0; j < 2; ++j) {
                  const __nv_bfloat16* src = !type ? p.ck : (p.cv ? p.cv + r * kDV + (8 * j + c) * 8
                                                                  : p.ck + r * kDQK + (8 * j + c) * 8);
                  cp_async16(Vt + j * kKB + tc::sw128(key, c), src, bytes);
                }
              }
            }
          }
        }
        if (nw > 0) {  // raw window tokens: contiguous rows
          const int64_t rw0 = srow[st][ne];
          const bool inb = CSA_INBOUNDS(rw0 >= 0 && rw0 + nw <= p.win_rows);
          for (int pc = pt; pc < nw * 24; pc += 256) {
            const int key = ne + pc / 24, c = pc % 24;
            cp_async16(Kt + (c >> 3) * kKB + tc::sw128(key, c & 7), inb ? p.wk + rw0 * kDQK + pc * 8 : p.q,
                       inb ? 16 : 0);
          }
          if (!SHV) {
            for (int pc = pt; pc < nw * 16; pc += 256) {
              const int key = ne + (pc >> 4), c = pc & 15;
              const __nv_bfloat16* src = p.wv ? p.wv + rw0 * kDV + pc * 8 : p.wk + (rw0 + (pc >> 4)) * kDQK + c * 8;
              cp_async16(Vt + (c >> 3) * kKB + tc::sw128(key, c & 7), src);
            }
          }
        }
        // slots past the end of the row: zero rows (their logits are masked)
        for (int pc = pt; pc < (kTcKeys - ne - nw) * 24; pc += 256) {
          const int key = ne + nw + pc / 24, c = pc % 24;
          cp_async16(Kt + (c >> 3) * kKB + tc::sw128(key, c & 7), p.q, 0);
        }
        if (!SHV) {
          for (int pc = pt; pc < (kTcKeys - ne - nw) * 16; pc += 256) {
            const int key = ne + nw + (pc >> 4), c = pc & 15;
            cp_async16(Vt + (c >> 3) * kKB + tc::sw128(key, c & 7), p.q, 0);
          }
        }
        cp_async_commit();
        sel_next = load_sel(tile + 1);
        if (FP8) {  // code * scale -> bf16 into the swizzled K (and V) tile; skipped slots get zeros
  #pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int key = (pt >> 3) + 32 * j, c = pt & 7;
            if (key >= ne) continue;
            const uint32_t w4[4] = {codes[j].x, codes[j].y, codes[j].z, codes[j].w};
            uint32_t outw[8];
  #pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t h01, h23;
              e4m3x4_to_f16x2x2(w4[q], h01, h23);
              const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
              const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
              outw[2 * q] = pack_bf16x2(f01.x * scl[j], f01.y * scl[j]);
              outw[2 * q + 1] = pack_bf16x2(f23.x * scl[j], f23.y * scl[j]);
            }
            const int blk = c >> 2;
            const uint4 lo = make_uint4(outw[0], outw[1], outw[2], outw[3]);
            const uint4 hi = make_uint4(outw[4], outw[5], outw[6], outw[7]);
            *reinterpret_cast<uint4*>(Kt + blk * kKB + tc::sw128(key, (2 * c) & 7)) = lo;
            *reinterpret_cast<uint4*>(Kt + blk * kKB + tc::sw128(key, (2 * c + 1) & 7)) = hi;
            if (!SHV) {
              *reinterpret_cast<uint4*>(Vt + blk * kKB + tc::sw128(key, (2 * c) & 7)) = lo;
              *reinterpret_cast<uint4*>(Vt + blk * kKB + tc::sw128(key, (2 * c + 1) & 7)) = hi;
            }
          }
        }
        cp_async_wait<0>();
        tc::fence_async_smem();
        named_sync(1, 256);
        if (pt == 0) bar_arrive(&full[st]);
      }
    }
  } else {
    // ===================== softmax: thread = key of the tile, 32 heads =====================
    // warp w: keys 32 (w % 4) .. +31 (its TMEM lane quarter), heads 32 (w / 4) .. +31
    const int key = (warp & 3) * 32 + lane;
    const int hb = (warp >> 2) * 32;
    for (int tile = 0; tile < ntiles; ++tile) {
      const int pb = tile & 1;
      if (healthy) healthy = tc::bar_wait(&sdone[pb], (tile >> 1) & 1);
      tc::fence_after_sync();
      float sv[32];
      tc::tmem_ld32(tmem + 64 * pb + lane_base + hb, sv);
      const bool valid = stype[tile & (kTypeRing - 1)][key] != 0;
      // sv <- logit x scale - running max (log2 units), one FMA per logit
      auto centre = [&]() {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(mref + hb + j);
          sv[j] = fmaf(sv[j], p.scale_log2, -m4.x);
          sv[j + 1] = fmaf(sv[j + 1], p.scale_log2, -m4.y);
          sv[j + 2] = fmaf(sv[j + 2], p.scale_log2, -m4.z);
          sv[j + 3] = fmaf(sv[j + 3], p.scale_log2, -m4.w);
        }
      };
      const bool trial = tile == 0;  // reference 0 for every head (see kFloorLog2)
      if (trial) {
        uint32_t seen = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          sv[j] *= p.scale_log2;
          seen |= (valid && sv[j] >= kFloorLog2) ? (1u << j) : 0u;
        }
        seen = __reduce_or_sync(0xffffffffu, seen);
        if (lane == 0 && seen) atomicOr(&hseen[hb >> 5], seen);
      } else {
        centre();
      }
      bool over = false;
#pragma unroll
      for (int j = 0; j < 32; ++j) over |= sv[j] > kRescaleLog2;
      bool need = named_sync_or(2, 256, over && valid);
      if (trial) need = need || (hseen[0] & hseen[1]) != 0xffffffffu;  // a head with no logit above the floor
      if (!need && trial && tid < 64) mref[tid] = 0.f;  // read after this tile's closing barrier
      if (need) {
        // new per-head maxima: this tile's maximum over its valid keys (the
        // reduction consumes sv; the logits are read again from TMEM below)
        tc::tmem_ld32(tmem + 64 * pb + lane_base + hb, sv);
#pragma unroll
        for (int j = 0; j < 32; ++j) sv[j] = valid ? sv[j] * p.scale_log2 : -INFINITY;
        const int h0 = warp_head_max32(sv, lane);
        wmax[warp & 3][hb + h0] = sv[0];
        named_sync(2, 256);
        if (tid < 64) {
          const float mo = mref[tid];
          const float mt = fmaxf(fmaxf(wmax[0][tid], wmax[1][tid]), fmaxf(wmax[2][tid], wmax[3][tid]));
          const float mn = fmaxf(mo, mt);
          corr_s[tid] = mo == -INFINITY ? 0.f : exp2f(mo - mn);
          mref[tid] = mn;
        }
        named_sync(2, 256);
        if (tile > 0) {  // O and l must be quiet: the previous tile's PV has to be done
          const int prev = tile - 1;
          if (healthy) healthy = tc::bar_wait(&empty[prev % NS], (prev / NS) & 1);
          tc::fence_after_sync();
#pragma unroll
          for (int c = 0; c < 2; ++c) {  // this thread's 32 columns of O^T, then of l^T
            const uint32_t ta = (c == 0 ? tO : tL) + lane_base + hb;
            float ov[32];
            tc::tmem_ld32(ta, ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= corr_s[hb + i];
            tc::tmem_st32(ta, ov);
          }
          tc::tmem_wait_st();
        }
        tc::tmem_ld32(tmem + 64 * pb + lane_base + hb, sv);
        centre();
      }
      // this key's P^T row, heads hb .. hb+31: four 16-byte chunks of the 128-byte swizzled row
      {
        uint8_t* Pb = Pst + pb * 16384;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float pv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) pv[u] = valid ? fast_exp2(sv[8 * c + u]) : 0.f;
          const uint4 v = make_uint4(pack_bf16x2(pv[0], pv[1]), pack_bf16x2(pv[2], pv[3]),
                                     pack_bf16x2(pv[4], pv[5]), pack_bf16x2(pv[6], pv[7]));
          *reinterpret_cast<uint4*>(Pb + tc::sw128(key, (hb >> 3) + c)) = v;
        }
      }
      tc::fence_async_smem();
      tc::fence_before_sync();
      named_sync(2, 256);
      if (tid == 0) bar_arrive(&pready[pb]);
    }
    if (ntiles > 0) {
      const int last = ntiles - 1;
      if (healthy) healthy = tc::bar_wait(&empty[last % NS], (last / NS) & 1);
      tc::fence_after_sync();
    }
  }
  cp_async_wait<0>();
  pdl_trigger();  // the epilogue is all that is left

  // ---- O^T (lane = channel) -> shared-memory transpose T[h][c] (fp32, in the P buffers), l per head ----
  float* T = reinterpret_cast<float*>(Pst);
  float* lrow = corr_s;  // l per head
  if (warp < 8) {
    const int c = (warp & 3) * 32 + lane, hb = (warp >> 2) * 32;
    float ov[32];
    if (ntiles > 0) {
      tc::tmem_ld32(tO + lane_base + hb, ov);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) ov[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) T[(hb + i) * kDV + c] = ov[i];
    if ((warp & 3) == 0) {  // every lane of l^T holds all 64 sums; lane 0 publishes this warp's 32
      float lv[32];
      if (ntiles > 0) {
        tc::tmem_ld32(tL + lane_base + hb, lv);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) lv[i] = 0.f;
      }
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) lrow[hb + i] = lv[i];
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 256);

  if (p.part != nullptr) {  // split record in global memory, merged by attn_merge_kernel
    for (int piece = tid; piece < 64 * 32; piece += kTcDecThreads) {
      const int hh = piece >> 5, q4 = piece & 31;
      float* rec = p.part + ((row * p.cl + split) * 64 + hh) * kRec;
      *reinterpret_cast<float4*>(rec + 4 * q4) = *reinterpret_cast<const float4*>(T + hh * kDV + 4 * q4);
    }
    if (tid < 64) {
      float* rec = p.part + ((row * p.cl + split) * 64 + tid) * kRec;
      *reinterpret_cast<float2*>(rec + kDV) = make_float2(mref[tid], lrow[tid]);
    }
    return;
  }
  if (p.cl == 1) {
    for (int piece = tid; piece < 64 * 16; piece += kTcDecThreads) {
      const int hh = piece >> 4, q8 = piece & 15;
      const float lh = lrow[hh];
      const float inv = lh > 0.f ? 1.f / lh : 0.f;
      const float* src = T + hh * kDV + 8 * q8;
      *reinterpret_cast<uint4*>(p.out + (row * p.H + hh) * kDV + 8 * q8) =
          make_uint4(pack_bf16x2(src[0] * inv, src[1] * inv), pack_bf16x2(src[2] * inv, src[3] * inv),
                     pack_bf16x2(src[4] * inv, src[5] * inv), pack_bf16x2(src[6] * inv, src[7] * inv));
    }
    if (tid < 64 && p.lse) {
      const float lh = lrow[tid];
      p.lse[row * p.H + tid] = lh > 0.f ? (mref[tid] + log2f(lh)) * kLn2 : -INFINITY;
    }
    return;
  }
  // cluster: records into the owner CTA's shared memory (head h is owned by rank h % cl)
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();  // peers may now write merge records over our Q/K tiles
  float* rbuf = reinterpret_cast<float*>(smem);
  for (int piece = tid; piece < 64 * 32; piece += kTcDecThreads) {
    const int hh = piece >> 5, q4 = piece & 31;
    float* dst = cluster.map_shared_rank(rbuf, hh % p.cl) + (static_cast<int64_t>(hh / p.cl) * p.cl + split) * kRec;
    *reinterpret_cast<float4*>(dst + 4 * q4) = *reinterpret_cast<const float4*>(T + hh * kDV + 4 * q4);
  }
  if (tid < 64) {
    float* dst = cluster.map_shared_rank(rbuf, tid % p.cl) + (static_cast<int64_t>(tid / p.cl) * p.cl + split) * kRec;
    dst[kDV] = mref[tid];
    dst[kDV + 1] = lrow[tid];
  }
  cluster.sync();
  const int sub = tid >> 5;  // warps 0-7, one head at a time each
  for (int j = sub; sub < 8 && split + j * p.cl < p.H; j += 8) {
    const int hh = split + j * p.cl;
    const float* rec = rbuf + static_cast<int64_t>(j) * p.cl * kRec;
    float M = -INFINITY;
    for (int c = 0; c < p.cl; ++c) M = fmaxf(M, rec[c * kRec + kDV]);
    const float bse = M == -INFINITY ? 0.f : M;
    float Lsum = 0.f, a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int c = 0; c < p.cl; ++c) {
      const float* r = rec + c * kRec;
      const float w = exp2f(r[kDV] - bse);
      Lsum += w * r[kDV + 1];
      const float4 u = *reinterpret_cast<const float4*>(r + lane * 4);
      a0 += w * u.x;
      a1 += w * u.y;
      a2 += w * u.z;
      a3 += w * u.w;
    }
    const float iv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    *reinterpret_cast<uint2*>(p.out + (row * p.H + hh) * kDV + lane * 4) =
        make_uint2(pack_bf16x2(a0 * iv, a1 * iv), pack_bf16x2(a2 * iv, a3 * iv));
    if (lane == 0 && p.lse) p.lse[row * p.H + hh] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
  }
}

// ---------------------------------------------------------------------------
// Query-blocked prefill (tcgen05): one CTA per block of QB = 256 / H
// consecutive queries, whose 256 (query, head) rows form two M = 128 MMA
// groups that share every staged key tile.  Consecutive queries see nearly
// the same keys, so the block's keys are staged once per 64-key tile and each
// row masks what its own query may not see:
//   dense (HCA): all visible entries [0, n) of the last query, then the raw
//     window run of the block; entry i needs (i+1)m - 1 <= t_q;
//   sparse (CSA, few heads): the union of the block's selected entries in
//     ascending order (built in shared memory from a per-entry bit set of
//     the queries that selected it), then the window run; a row sees an
//     entry slot iff its query selected that entry;
//   window token p: t_q - w_s < p <= t_q.
// Warps 0-3 own rows 0-127 (group 0), warps 4-7 rows 128-255 (group 1): one
// thread per row, in its TMEM lane.  Warps 8-10 copy tiles with cp.async
// whose completions arrive on the stage barrier (the copying threads never
// wait for their data); one thread of warp 11 issues every MMA (twelve warps:
// three per SM sub-partition, so that each thread may hold 168 registers):
//   S_g = Q_g K^T   (M = 128 rows, N = 64 keys, K = 192), double-buffered;
//   O_g += P_g V    (M = 128 rows, N = 128 channels, K = 64 keys).
// TMEM: S[g][buf] in columns 64 (2g + buf), O_g in 256 + 128 g.
// ---------------------------------------------------------------------------
constexpr int kQbKeys = 64;
constexpr int kQbThreads = 384;
constexpr int kQbLoaders = 96;  // warps 8-10
constexpr int kQbMaxCand = 2048;   // sparse path: block queries x k
constexpr int kQbMaxEnt = 16384;   // sparse path: entries per sequence (bit set in the P buffers)

struct QbLayout {
  size_t q, k, v, p, ulist, qbits, bars, total;
};

__host__ __device__ inline QbLayout qb_layout() {
  QbLayout L;
  size_t off = 0;
  L.q = off; off += 2 * 3 * 16384;      // Q: 2 groups x 3 blocks of 128 rows x 128 B
  L.k = off; off += 2 * 3 * 8192;       // K: 2 stages x 64 keys x 192 dims
  L.v = off; off += 2 * 2 * 8192;       // V: 2 stages x 64 keys x 128 dims
  L.p = off; off += 2 * 16384;          // P: 2 groups x 128 rows x 64 keys (prologue: entry bit set)
  L.ulist = off; off += kQbMaxCand * 2; // union entries (uint16)
  L.qbits = off; off += 16 * kQbMaxCand / 8;  // per query: bit u = it selected union entry u
  L.bars = off; off += 256;              // 19 mbarriers + the TMEM address
  L.total = off + 1024;
  return L;
}

// Bits of the slots [lo, hi] (inclusive) within the 64-slot tile starting at sb.
__device__ __forceinline__ uint64_t range_bits(int lo, int hi, int sb) {
  const int a = lo - sb > 0 ? lo - sb : 0;
  const int b = hi + 1 - sb < 64 ? hi + 1 - sb : 64;
  if (a >= b) return 0ull;
  const uint64_t upto = b == 64 ? ~0ull : ((1ull << b) - 1ull);
  return upto & ~((1ull << a) - 1ull);
}

// Geometry of one query block.
struct QbBlock {
  int64_t b, r0, t0, tl, wlo0, nwin;
  int nq;
};
// a / b for a >= 0, b > 0: a 32-bit division when both fit (the 64-bit one is
// emulated and costs more than the rest of a block's geometry)
__device__ __forceinline__ int64_t qb_div(int64_t a, int64_t b) {
  if (((a | b) >> 32) == 0) return static_cast<uint32_t>(a) / static_cast<uint32_t>(b);
  return a / b;
}
__device__ __forceinline__ QbBlock qb_block(const AttnParams& p, int64_t blk) {
  const int QB = 256 / p.H;
  const int64_t nblk = (p.Tq + QB - 1) / QB;
  QbBlock k;
  k.b = qb_div(blk, nblk);
  k.r0 = (blk - k.b * nblk) * QB;  // first query row of the block within its sequence
  k.nq = static_cast<int>((p.Tq - k.r0) < QB ? (p.Tq - k.r0) : QB);
  k.t0 = p.q_pos0 + k.r0;
  k.tl = k.t0 + k.nq - 1;
  k.wlo0 = (k.t0 - p.wlen + 1) > 0 ? (k.t0 - p.wlen + 1) : 0;
  k.nwin = p.wlen > 0 ? (k.tl - k.wlo0 + 1) : 0;
  return k;
}
// Dense entry run of a block: the entries visible to its last query.
__device__ __forceinline__ int64_t qb_dense_entries(const AttnParams& p, const QbBlock& k) {
  const int64_t n = qb_div(k.tl + 1, p.stride);
  return n < p.N ? n : p.N;
}

// Dense blocks run persistently: CTA c takes blocks c, c + gridDim.x, ...,
// and its pipeline carries over from one block to the next (the copies of the
// next block's key tiles start as soon as stages free up, its queries as soon
// as the last S of the current block is done, and its first S while the
// current block's last tile drains).  Stage and TMEM-buffer parities follow
// a tile counter that runs across the CTA's blocks.  Sparse blocks (which
// build their union with whole-CTA barriers) run one block per CTA.
__global__ void __launch_bounds__(kQbThreads, 1) attn_qblock_kernel(AttnParams p,
                                                                    const __grid_constant__ CUtensorMap qmap) {
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const QbLayout L = qb_layout();
  uint8_t* Qs = smem + L.q;
  uint8_t* Kst = smem + L.k;
  uint8_t* Vst = smem + L.v;
  uint8_t* Pst = smem + L.p;
  uint16_t* ulist = reinterpret_cast<uint16_t*>(smem + L.ulist);
  uint32_t* qbits = reinterpret_cast<uint32_t*>(smem + L.qbits);  // [16 queries][kQbMaxCand / 32]
  uint64_t* kfull = reinterpret_cast<uint64_t*>(smem + L.bars);  // [2] K stage loaded (one arrival per loader)
  uint64_t* vfull = kfull + 2;                                     // [2] V stage loaded (same)
  uint64_t* kfree = vfull + 2;                                     // [2] both S of the K stage's tile done
  uint64_t* vfree = kfree + 2;                                     // [2] both PV of the V stage's tile done
  uint64_t* sdone = vfree + 2;                                     // [2 groups][2 bufs] S done
  uint64_t* pready = sdone + 4;                                    // [2 groups] P written
  uint64_t* pvdone = pready + 2;                                   // [2 groups] PV done
  uint64_t* qfull = pvdone + 2;                                    // the block's queries landed
  uint64_t* qfree = qfull + 1;                                     // the block's last S done (Q may be replaced)
  uint64_t* ofree = qfree + 1;                                     // [2 groups] O read out by the epilogue
  uint32_t* tslot = reinterpret_cast<uint32_t*>(ofree + 2);
  __shared__ int s_count[kQbThreads / 32];
  __shared__ int s_union;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H;
  const bool sparse = p.idx != nullptr;
  const int64_t nblocks = p.qb_blocks;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) tc::bar_init(&kfull[i], kQbLoaders);  // kfull, vfull
    for (int i = 4; i < 16; ++i) tc::bar_init(&kfull[i], 1);
    tc::bar_init(qfull, 1);
    tc::bar_init(qfree, 1);
    tc::bar_init(&ofree[0], 1);
    tc::bar_init(&ofree[1], 1);
    tc::bar_init_fence();
  }
  __syncthreads();  // the barriers exist before any copy arrives on one
  if (warp == 0) tc::tmem_alloc(tslot, 512);

  // queries of a block (one thread): rows (query, head) of both groups, six
  // TMA boxes of 128 rows x 64 dims in the 128-byte swizzle (the [B][Tq*H][192]
  // tensor map zero-fills the rows past the sequence's last query)
  auto load_q = [&](const QbBlock& k) {  // (read once: evict first, so the key rows stay in L2)
    tc::bar_arrive_expect_tx(qfull, 6 * 16384);
    const int y0 = static_cast<int>(k.r0 * H);
    const uint64_t pol = tc::l2_evict_first_policy();
    for (int g = 0; g < 2; ++g)
      for (int cb = 0; cb < 3; ++cb)
        tc::tma_load_3d_stream(Qs + g * 49152 + cb * 16384, &qmap, 64 * cb, y0 + 128 * g, static_cast<int>(k.b),
                               qfull, pol);
  };

  // sparse: the union of the block's selections (one block per CTA)
  int64_t n_ent_sparse = 0;
  if (sparse) {
    const QbBlock k = qb_block(p, blockIdx.x);
    if (tid == 8 * 32) load_q(k);  // waited for by the MMA thread only
    // per-entry bit set of the block's queries that selected it (16 bits per entry, in the P buffers)
    uint32_t* bits = reinterpret_cast<uint32_t*>(Pst);
    const int nwords = static_cast<int>((p.N + 1) / 2);
    for (int w = tid; w < nwords; w += kQbThreads) bits[w] = 0u;
    for (int w = tid; w < 16 * kQbMaxCand / 32; w += kQbThreads) qbits[w] = 0u;
    __syncthreads();
    for (int c = tid; c < k.nq * p.k; c += kQbThreads) {
      const int q = c / p.k;
      const int64_t tq = k.t0 + q;
      const int64_t i = __ldg(p.idx + (k.b * p.Tq + k.r0 + q) * p.k + (c % p.k));
      if (i >= 0 && i < p.N && (i + 1) * p.stride - 1 <= tq)
        atomicOr(&bits[i >> 1], 1u << (static_cast<int>(i & 1) * 16 + q));
    }
    __syncthreads();
    // ascending compaction: thread chunks of words, counts, a block scan, then the writes
    const int per = (nwords + kQbThreads - 1) / kQbThreads;
    const int w0 = tid * per, w1 = (w0 + per) < nwords ? (w0 + per) : nwords;
    int cnt = 0;
    for (int w = w0; w < w1; ++w) {
      const uint32_t v = bits[w];
      cnt += ((v & 0xffffu) != 0u) + ((v >> 16) != 0u);
    }
    int incl = cnt;  // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_count[warp] = incl;
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int w = 0; w < kQbThreads / 32; ++w) {
        const int c2 = s_count[w];
        s_count[w] = run;
        run += c2;
      }
      s_union = run;
    }
    __syncthreads();
    int pos = s_count[warp] + incl - cnt;
    auto put = [&](int e, uint32_t qm) {  // union entry `pos`: entry e, selected by the queries in qm
      ulist[pos] = static_cast<uint16_t>(e);
      for (; qm != 0u; qm &= qm - 1u) atomicOr(&qbits[(__ffs(qm) - 1) * (kQbMaxCand / 32) + (pos >> 5)], 1u << (pos & 31));
      ++pos;
    };
    for (int w = w0; w < w1; ++w) {
      const uint32_t v = bits[w];
      if ((v & 0xffffu) != 0u) put(2 * w, v & 0xffffu);
      if ((v >> 16) != 0u) put(2 * w + 1, v >> 16);
    }
    n_ent_sparse = s_union;
  }
  tc::fence_before_sync();
  __syncthreads();  // the union is ready and the P buffers are free again (Q may still be landing)
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;
  bool healthy = true;
  // this CTA's blocks: one (sparse), or every gridDim.x-th (dense)
  const int64_t blk_step = sparse ? nblocks : gridDim.x;
  auto n_entries = [&](const QbBlock& k) { return sparse ? n_ent_sparse : qb_dense_entries(p, k); };

  if (warp >= 8 && warp < 11) {
    // ===================== producer: cp.async copies that arrive by themselves =====================
    const __nv_bfloat16* ve = p.cv ? p.cv : p.ck;
    const int ves = p.cv ? kDV : kDQK;
    const __nv_bfloat16* vw = p.wv ? p.wv : p.wk;
    const int vws = p.wv ? kDV : kDQK;
    const int pw = warp - 8, c8 = lane & 7;
    int64_t gt = 0;  // tiles of this CTA's earlier blocks
    int jq = 0;      // earlier blocks that had tiles (each loaded its queries once)
    for (int64_t blk = blockIdx.x; blk < nblocks && healthy; blk += blk_step) {
      const QbBlock k = qb_block(p, blk);
      const int64_t n_ent = n_entries(k);
      const int64_t n_slots = n_ent + k.nwin;
      const int ntiles = static_cast<int>((n_slots + kQbKeys - 1) / kQbKeys);
      if (ntiles == 0) continue;
      const int64_t ebase = k.b * p.N;
      const int64_t wbase = k.b * p.wrows - p.wpos0 + k.wlo0;
      // K (three 128-byte blocks per key) or V (two) of one tile: eight lanes per
      // 128-byte row segment, four keys per warp instruction
      auto issue = [&](bool is_k, uint8_t* T, int tile) {
        const int64_t a0 = static_cast<int64_t>(tile) * kQbKeys;
        for (int key = pw * 4 + (lane >> 3); key < kQbKeys; key += 12) {
          const int64_t sl = a0 + key;
          const __nv_bfloat16* src = nullptr;
          if (sl < n_ent) {
            const int64_t e = ebase + (sparse ? static_cast<int64_t>(ulist[sl]) : sl);
            if (CSA_INBOUNDS(e >= 0 && e < p.ent_rows)) src = is_k ? p.ck + e * kDQK : ve + e * ves;
          } else if (sl < n_slots) {
            const int64_t w = wbase + (sl - n_ent);
            if (CSA_INBOUNDS(w >= 0 && w < p.win_rows)) src = is_k ? p.wk + w * kDQK : vw + w * vws;
          }
          uint8_t* dst = T + tc::sw128(key, c8);
          const __nv_bfloat16* s8 = src != nullptr ? src + c8 * 8 : p.q;
          const int bytes = src != nullptr ? 16 : 0;
          cp_async16(dst, s8, bytes);
          cp_async16(dst + 8192, src != nullptr ? s8 + 64 : p.q, bytes);
          if (is_k) cp_async16(dst + 16384, src != nullptr ? s8 + 128 : p.q, bytes);
        }
      };
      auto wait_free = [&](uint64_t* bar, uint32_t parity) {  // warp-uniform outcome
        bool ok = true;
        if (lane == 0) ok = tc::bar_wait(bar, parity);
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      };
      // K(t) is issued before V(t - 1): K stages are freed when both S are done,
      // V stages when both PV are (stage and parity from the CTA-wide tile count);
      // a dense block's queries follow its first K tile, once the previous
      // block's last S is done
      for (int it = 0; it <= ntiles; ++it) {
        if (it < ntiles) {
          const int64_t G = gt + it;
          const int st = static_cast<int>(G & 1);
          if (G >= 2 && !wait_free(&kfree[st], static_cast<uint32_t>(((G >> 1) - 1) & 1))) {
            healthy = false;
            break;
          }
          issue(true, Kst + st * 3 * 8192, it);
          cp_async_mbar_arrive_noinc(&kfull[st]);
        }
        if (it == 0 && !sparse) {
          if (jq > 0 && !wait_free(qfree, (jq - 1) & 1)) {
            healthy = false;
            break;
          }
          if (tid == 8 * 32) load_q(k);
        }
        if (it >= 1) {
          const int64_t G = gt + it - 1;
          const int st = static_cast<int>(G & 1);
          if (G >= 2 && !wait_free(&vfree[st], static_cast<uint32_t>(((G >> 1) - 1) & 1))) {
            healthy = false;
            break;
          }
          issue(false, Vst + st * 2 * 8192, it - 1);
          cp_async_mbar_arrive_noinc(&vfull[st]);
        }
      }
      gt += ntiles;
      ++jq;
    }
    cp_async_wait<0>();
  } else if (warp == 11) {
    // ===================== MMA issue (one thread) =====================
    constexpr uint32_t kIdescS = tc::idesc_bf16(128, kQbKeys, false);
    constexpr uint32_t kIdescO = tc::idesc_bf16(128, kDV, true);
    if (lane == 0) {
      int64_t gt = 0;
      int jq = 0;
      for (int64_t blk = blockIdx.x; blk < nblocks && healthy; blk += blk_step) {
        const QbBlock k = qb_block(p, blk);
        const int64_t n_slots = n_entries(k) + k.nwin;
        const int ntiles = static_cast<int>((n_slots + kQbKeys - 1) / kQbKeys);
        if (ntiles == 0) continue;
        auto issue_s = [&](int tile) {  // S of both groups for the block's tile; the last one frees Q
          const int64_t G = gt + tile;
          const int st = static_cast<int>(G & 1);
          if (healthy) healthy = tc::bar_wait(&kfull[st], static_cast<uint32_t>((G >> 1) & 1));
          const uint32_t ka = smem_u32(Kst + st * 3 * 8192);
          tc::fence_async_smem();  // the stage was written by cp.async
          tc::fence_after_sync();
          for (int g = 0; g < 2; ++g) {
            const uint32_t qa = smem_u32(Qs + g * 49152);
#pragma unroll
            for (int kk = 0; kk < 12; ++kk)
              tc::mma_bf16_ss(tmem + 64 * (2 * g + st), tc::desc_sw128(qa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                              tc::desc_sw128(ka + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), kIdescS,
                              kk > 0 ? 1u : 0u);
            tc::mma_commit(&sdone[2 * g + st]);
          }
          tc::mma_commit(&kfree[st]);
          if (tile == ntiles - 1) tc::mma_commit(qfree);
        };
        if (healthy) healthy = tc::bar_wait(qfull, static_cast<uint32_t>(jq & 1));
        for (int tt = 0; tt < 2 && tt < ntiles; ++tt) issue_s(tt);
        for (int tile = 0; tile < ntiles; ++tile) {
          const int64_t G = gt + tile;
          const int st = static_cast<int>(G & 1);
          const uint32_t va = smem_u32(Vst + st * 2 * 8192);
          for (int g = 0; g < 2; ++g) {
            if (healthy) healthy = tc::bar_wait(&pready[g], static_cast<uint32_t>(G & 1));
            if (tile == 0 && jq > 0 && healthy)  // the previous block's O of this group has been read out
              healthy = tc::bar_wait(&ofree[g], static_cast<uint32_t>((jq - 1) & 1));
            if (g == 0 && healthy) {
              healthy = tc::bar_wait(&vfull[st], static_cast<uint32_t>((G >> 1) & 1));
              tc::fence_async_smem();  // the stage was written by cp.async
            }
            tc::fence_after_sync();
            const uint32_t pa = smem_u32(Pst + g * 16384);
#pragma unroll
            for (int ks = 0; ks < kQbKeys / 16; ++ks)
              tc::mma_bf16_ss(tmem + 256 + 128 * g, tc::desc_sw128(pa + ks * 32, 16, 1024),
                              tc::desc_sw128(va + ks * 2048, 8192, 1024), kIdescO, (tile > 0 || ks > 0) ? 1u : 0u);
            tc::mma_commit(&pvdone[g]);
          }
          tc::mma_commit(&vfree[st]);
          if (tile + 2 < ntiles) issue_s(tile + 2);
        }
        gt += ntiles;
        ++jq;
      }
    }
  } else if (warp < 8) {
    // ===================== softmax: thread = row (query, head) of group g =====================
    const int g = warp >> 2;
    const int rl = tid & 127;          // TMEM lane
    const int r = 128 * g + rl;        // row of the block
    const int qr = r / H;              // query of this row within the block
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + 256 + 128 * g;
    int64_t gt = 0;
    for (int64_t blk = blockIdx.x; blk < nblocks; blk += blk_step) {
      const QbBlock k = qb_block(p, blk);
      const int64_t n_ent = n_entries(k);
      const int64_t n_slots = n_ent + k.nwin;
      const int ntiles = static_cast<int>((n_slots + kQbKeys - 1) / kQbKeys);
      const bool row_ok = qr < k.nq;
      // this row's output (the block geometry is not needed past this point)
      const int64_t orow = (k.b * p.Tq + k.r0) * H + r;
      const int64_t tq = k.t0 + (row_ok ? qr : 0);
      int64_t nv_q = qb_div(tq + 1, p.stride);
      if (nv_q > p.N) nv_q = p.N;
      const int64_t lo_q = (tq - p.wlen + 1) > 0 ? (tq - p.wlen + 1) : 0;
      // slot numbers (below 2^31): the entry run, this row's visible entries and window slots
      const int ent32 = static_cast<int>(n_ent), nv32 = static_cast<int>(nv_q);
      const int wv_lo = static_cast<int>(n_ent + (lo_q - k.wlo0)), wv_hi = static_cast<int>(n_ent + (tq - k.wlo0));
      float m_ref = -INFINITY, l = 0.f;
      for (int tile = 0; tile < ntiles; ++tile) {
        const int64_t G = gt + tile;
        const int st = static_cast<int>(G & 1);
        if (healthy) healthy = tc::bar_wait(&sdone[2 * g + st], static_cast<uint32_t>((G >> 1) & 1));
        tc::fence_after_sync();
        float sv[kQbKeys];
        tc::tmem_ld32(tmem + 64 * (2 * g + st) + lane_base, sv);
        tc::tmem_ld32(tmem + 64 * (2 * g + st) + lane_base + 32, sv + 32);
        // this row's visible slots of the tile as a bit mask: its entries, then its window run
        const int sb = tile * kQbKeys;
        uint64_t vm = 0;
        if (row_ok) {
          if (sb < ent32) {
            vm = sparse ? (static_cast<uint64_t>(qbits[qr * (kQbMaxCand / 32) + (sb >> 5) + 1]) << 32) |
                              qbits[qr * (kQbMaxCand / 32) + (sb >> 5)]
                        : range_bits(0, nv32 - 1, sb);
            vm &= range_bits(0, ent32 - 1, sb);
          }
          vm |= range_bits(wv_lo, wv_hi, sb);
        }
        const uint32_t vlo = static_cast<uint32_t>(vm), vhi = static_cast<uint32_t>(vm >> 32);
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < kQbKeys; ++j) {
          const bool ok = (((j < 32 ? vlo : vhi) >> (j & 31)) & 1u) != 0u;
          sv[j] = ok ? sv[j] * p.scale_log2 : -INFINITY;
          mx = fmaxf(mx, sv[j]);
        }
        const float m_new = fmaxf(m_ref, mx);
        const bool resc = m_new > m_ref + 8.f;
        float corr = 1.f;
        if (resc) {
          corr = exp2f(m_ref - m_new);
          m_ref = m_new;
          l *= corr;
        }
        const float base = m_ref == -INFINITY ? 0.f : m_ref;
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < kQbKeys; ++j) {
          sv[j] = fast_exp2(sv[j] - base);
          sum += sv[j];
        }
        l += sum;
        if (tile > 0) {  // PV of the previous tile: the P buffer is free and O is quiet
          if (healthy) healthy = tc::bar_wait(&pvdone[g], static_cast<uint32_t>((G - 1) & 1));
          tc::fence_after_sync();
          if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float ov[32];
              tc::tmem_ld32(tO + lane_base + 32 * c, ov);
#pragma unroll
              for (int i = 0; i < 32; ++i) ov[i] *= corr;
              tc::tmem_st32(tO + lane_base + 32 * c, ov);
            }
            tc::tmem_wait_st();
          }
        }
        {
          uint8_t* Pb = Pst + g * 16384;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = make_uint4(pack_bf16x2(sv[8 * c], sv[8 * c + 1]), pack_bf16x2(sv[8 * c + 2], sv[8 * c + 3]),
                                       pack_bf16x2(sv[8 * c + 4], sv[8 * c + 5]),
                                       pack_bf16x2(sv[8 * c + 6], sv[8 * c + 7]));
            *reinterpret_cast<uint4*>(Pb + tc::sw128(rl, c)) = v;
          }
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        named_sync(2 + g, 128);
        if (rl == 0) bar_arrive(&pready[g]);
      }
      if (ntiles > 0 && healthy) healthy = tc::bar_wait(&pvdone[g], static_cast<uint32_t>((gt + ntiles - 1) & 1));
      tc::fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint32_t ob[4][16];  // the normalised row, bf16 pairs
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float ov[32];
        if (ntiles > 0) {
          tc::tmem_ld32(tO + lane_base + 32 * c, ov);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) ob[c][i] = pack_bf16x2(ov[2 * i] * inv, ov[2 * i + 1] * inv);
      }
      if (ntiles > 0) {  // O is read out: the next block's first PV may overwrite it
        tc::fence_before_sync();
        named_sync(2 + g, 128);
        if (rl == 0) bar_arrive(&ofree[g]);
      }
      if (row_ok) {
        __nv_bfloat16* o = p.out + orow * kDV;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            __stcs(reinterpret_cast<uint4*>(o + 32 * c + 2 * i),  // streamed out: not kept in L2
                   make_uint4(ob[c][i], ob[c][i + 1], ob[c][i + 2], ob[c][i + 3]));
        }
        if (p.lse) p.lse[orow] = l > 0.f ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
      }
      gt += ntiles;
    }
  }
  pdl_trigger();
  cp_async_wait<0>();  // (the query copies landed long before; nothing of this thread stays in flight)
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Merge of the split records of each (row, head): one warp per head, four
// channels per lane.  out = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c with
// M = max_c m_c; lse = ln 2 (M + log2 sum_c 2^(m_c - M) l_c).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) attn_merge_kernel(const float* __restrict__ part, int nsplit, int H,
                                                         __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  pdl_wait();  // (no early trigger: the next kernel is usually a long one)
  const int lane = threadIdx.x & 31;
  const int64_t rh = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);  // row * H + head
  const int64_t row = rh / H;
  const int hh = static_cast<int>(rh % H);
  const float* rec0 = part + (row * nsplit * H + hh) * kRec;
  const int64_t cstride = static_cast<int64_t>(H) * kRec;
  // batches of up to 24 split records, all of a batch's loads in flight at
  // once (one batch for up to 24 splits), merged online across batches
  constexpr int kBatch = 24;
  float M = -INFINITY, Lsum = 0.f;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = 0; c0 < nsplit; c0 += kBatch) {
    float2 ml[kBatch];
    float4 u[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const bool ok = c0 + j < nsplit;
      const float* r = rec0 + (ok ? c0 + j : 0) * cstride;
      ml[j] = ok ? __ldg(reinterpret_cast<const float2*>(r + kDV)) : make_float2(-INFINITY, 0.f);
      u[j] = ok ? __ldg(reinterpret_cast<const float4*>(r) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mb = -INFINITY;
#pragma unroll
    for (int j = 0; j < kBatch; ++j) mb = fmaxf(mb, ml[j].x);
    const float mn = fmaxf(M, mb);
    if (mn != -INFINITY && M != mn) {  // rescale what earlier batches summed
      const float f = M == -INFINITY ? 0.f : exp2f(M - mn);
      Lsum *= f;
      a.x *= f;
      a.y *= f;
      a.z *= f;
      a.w *= f;
      M = mn;
    }
    const float bse = M == -INFINITY ? 0.f : M;
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const float w = exp2f(ml[j].x - bse);
      Lsum += w * ml[j].y;
      a.x += w * u[j].x;
      a.y += w * u[j].y;
      a.z += w * u[j].z;
      a.w += w * u[j].w;
    }
  }
  const float iv = Lsum > 0.f ? 1.f / Lsum : 0.f;
  *reinterpret_cast<uint2*>(out + rh * kDV + lane * 4) =
      make_uint2(pack_bf16x2(a.x * iv, a.y * iv), pack_bf16x2(a.z * iv, a.w * iv));
  if (lane == 0 && lse) lse[rh] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
}

// ---------------------------------------------------------------------------
// Expiring wait (failure-detection check): one thread waits, through the same
// bounded wait every kernel of the library uses, on an mbarrier that nothing
// arrives at.  The wait runs out after `limit` rounds and records the timeout
// in this unit's error word.  No copy, MMA or TMEM allocation is involved.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) wait_expire_kernel(uint32_t limit) {
  pdl_wait();
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::bar_init(&bar, 1);
    tc::bar_init_fence();
    tc::bar_wait_bounded(&bar, 0, limit);  // phase 0 never completes: no arrival
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// Splits of a row's slots for the tcgen05 kernel (one CTA per SM): rows that
// cannot fill the `sms` SMs by themselves are split so that all rows' CTAs
// run in one wave; the splits then merge through global-memory records.
struct TcSplit {
  int nsplit, tps;
};
TcSplit tc_split(int64_t R, int64_t max_slots, int64_t sms) {
  const int64_t tiles = max_slots > 0 ? (max_slots + kTcKeys - 1) / kTcKeys : 1;
  int64_t ns = R >= sms ? 1 : sms / R;
  if (ns < 1) ns = 1;
  if (ns > tiles) ns = tiles;
  const int64_t tps = (tiles + ns - 1) / ns;
  ns = (tiles + tps - 1) / tps;
  return TcSplit{static_cast<int>(ns), static_cast<int>(tps)};
}
size_t tc_part_bytes(int64_t R, int H, int64_t max_slots) {
  if (H != 64 || R <= 0) return 0;
  const TcSplit sp = tc_split(R, max_slots, num_sms());
  return sp.nsplit > 1 ? static_cast<size_t>(R) * sp.nsplit * H * kRec * sizeof(float) : 0;
}

struct Plan {
  int cl, tps;
};

Plan plan(int64_t R, int64_t max_slots, int tile_keys) {
  const int64_t tiles = max_slots > 0 ? (max_slots + tile_keys - 1) / tile_keys : 1;
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

using TcKernelFn = void (*)(AttnParams);

TcKernelFn pick_tc(bool fp8, bool shv) {
  if (fp8) return attn_tc_kernel<true, true>;  // (an FP8 cache with a separate V never takes this path)
  return shv ? attn_tc_kernel<false, true> : attn_tc_kernel<false, false>;
}

size_t smem_bytes(bool use_tc, bool fp8, bool shv, int tps) {
  return use_tc ? tc_layout(fp8, shv, tps).total : smem_layout(fp8, shv, tps).total;
}

// Clusters of this kernel (cluster size cl, given shared memory and block size)
// the device can keep resident at once; 0 if it cannot run them at all.
template <typename Fn>
int max_active_clusters(Fn fn, int cl, size_t smem, int threads) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, int, size_t, int>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(dev, reinterpret_cast<const void*>(fn), cl, smem, threads);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cl));
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = cl;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache[key] = n;
  return n;
}

// Cluster size for `rows` rows of `tiles` tiles each: the largest size <= want
// whose clusters all fit on the device at once (one wave); if none does, the
// largest size that runs at all.
template <typename Fn>
int choose_cluster(Fn fn, int want, int64_t rows, size_t smem, int threads) {
  int fallback = 1;
  for (int cl = want; cl > 1; --cl) {
    const int n = max_active_clusters(fn, cl, smem, threads);
    if (n >= rows) return cl;
    if (n > 0 && fallback == 1) fallback = cl;
  }
  return fallback;
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
               float scale, void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream,
               const csa_packed* pk = nullptr, int32_t max_sms = 0) {
  clear_error();
  CSA_REQUIRE(B >= 0 && Tq >= 0, "%s: negative size", name);
  CSA_REQUIRE(H == 16 || H == 64, "%s: H must be 16 or 64 (got %d)", name, H);
  CSA_REQUIRE(stride >= 1, "%s: stride must be >= 1", name);
  CSA_REQUIRE(q_pos0 >= 0, "%s: q_pos0 must be >= 0", name);
  CSA_REQUIRE(scale == scale && scale > -3.0e38f && scale < 3.0e38f, "%s: scale must be finite", name);
  if (csa_status st = check_cache(name, cache); st != CSA_OK) return st;
  CSA_REQUIRE(q_pos0 < (int64_t(1) << 50), "%s: q_pos0 must be below 2^50", name);
  // bound both factors before multiplying so that B * Tq cannot overflow
  constexpr int64_t kRowLim = (int64_t(1) << 31) / kMaxCluster;
  CSA_REQUIRE(B < kRowLim && Tq < kRowLim && (Tq == 0 || B <= (kRowLim - 1) / Tq), "%s: too many query rows",
              name);
  const int64_t R = B * Tq;
  if (R == 0) return CSA_OK;
  CSA_REQUIRE_PTR(q);
  CSA_REQUIRE_PTR(out);
  CSA_REQUIRE(lse == nullptr || (reinterpret_cast<uintptr_t>(lse) & 3u) == 0, "%s: lse misaligned", name);
  if (idx) CSA_REQUIRE(k >= 1 && k <= 4096 && aligned16(idx), "%s: idx misaligned or k out of [1, 4096]", name);
  int wlen = 0;
  if (win) {
    CSA_REQUIRE(win->reserved == 0 && win->len >= 0, "%s: bad window descriptor", name);
    wlen = win->len;
  }
  if (pk != nullptr) {
    CSA_REQUIRE(pk->cu_tokens != nullptr && pk->cu_entries != nullptr && pk->n_seqs > 0,
                "%s: packed offsets NULL or no sequences", name);
    CSA_REQUIRE(cache->n_entries == pk->total_entries, "%s: cache->n_entries must equal packed->total_entries",
                name);
    CSA_REQUIRE(wlen == 0 || (win->pos0 == 0 && win->rows == pk->total_tokens),
                "%s: with packed sequences the window buffer is the packed tokens (pos0 0, rows total_tokens)",
                name);
  }
  if (wlen > 0) {
    CSA_REQUIRE(win->k && aligned16(win->k), "%s: win->k NULL or misaligned", name);
    CSA_REQUIRE(!win->v || aligned16(win->v), "%s: win->v misaligned", name);
  }
  if (wlen > 0 && pk == nullptr) {
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
  // slots of the longest row: k + window for CSA; for HCA every entry of the (longest) sequence + window
  const int64_t n_dense = pk != nullptr ? (static_cast<int64_t>(pk->max_tokens) + stride - 1) / stride : N;
  const int64_t max_slots = (idx ? k : n_dense) + wlen;
  // tcgen05 path for 64 heads; H = 16, and an FP8 cache combined with a separate
  // raw-window V (too much shared memory for the staged tiles), use the warp-MMA kernel
  const bool use_tc = H == 64 && !(fp8 && !shv);
  const int tile_keys = use_tc ? kTcKeys : kKeys;
  Plan pl = plan(R, max_slots, tile_keys);
  float* part = nullptr;
  bool tc_cluster = false;  // tcgen05 path: splits merged in a cluster (else through global records)
  if (use_tc && !ensure_smem(reinterpret_cast<const void*>(pick_tc(fp8, shv)),
                             static_cast<int>(tc_layout(fp8, shv, 0).total)))
    return fail(CSA_ERR_CUDA, "%s: cannot raise the shared memory limit", name);
  if (use_tc) {
    // an SM budget (work beside this call on another stream keeps the rest)
    // bounds the splits; it takes the global-record merge, whose split count
    // follows the budget exactly
    const int64_t sms = (max_sms > 0 && max_sms < num_sms()) ? max_sms : num_sms();
    const TcSplit sp = tc_split(R, max_slots, sms);
    if (sp.nsplit > 1 && pl.cl > 1 && max_sms <= 0) {
      // A cluster merge (distributed shared memory, no second kernel) wins when
      // a co-resident cluster size leaves no more tiles per CTA than the global
      // split does; with even one tile more per CTA the split and its one-round
      // merge kernel are faster (8 CSA decode rows of 17 tiles: 9-CTA clusters
      // of 2 tiles 12.1 us, 17 CTAs of 1 tile + merge 11.4 us, graph-replayed).
      static std::mutex mu;
      bool nonportable = true;
      {
        std::lock_guard<std::mutex> lock(mu);
        const TcKernelFn f = pick_tc(fp8, shv);
        if (cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
          cudaGetLastError();
          nonportable = false;
        }
      }
      const int want = nonportable ? pl.cl : (pl.cl > 8 ? 8 : pl.cl);
      const int cl = choose_cluster(pick_tc(fp8, shv), want, R, tc_layout(fp8, shv, 0).total, kTcDecThreads);
      const int64_t tiles = max_slots > 0 ? (max_slots + kTcKeys - 1) / kTcKeys : 1;
      const int64_t tps = (tiles + cl - 1) / cl;
      if (cl > 1 && max_active_clusters(pick_tc(fp8, shv), cl, tc_layout(fp8, shv, 0).total, kTcDecThreads) >= R &&
          tps <= sp.tps) {
        tc_cluster = true;
        pl.tps = static_cast<int>(tps);
        pl.cl = static_cast<int>((tiles + tps - 1) / tps);
      }
    }
    if (!tc_cluster) {
      pl.cl = sp.nsplit;
      pl.tps = sp.tps;
    }
    if (!tc_cluster && sp.nsplit > 1) {
      const size_t need = tc_part_bytes(R, H, max_slots);
      if (workspace == nullptr || workspace_bytes < need)
        return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed (got %zu)", name, need, workspace_bytes);
      CSA_REQUIRE(aligned16(workspace), "%s: workspace is not 16-byte aligned", name);
      part = static_cast<float*>(workspace);
    }
  }
  const TcKernelFn tfn = use_tc ? pick_tc(fp8, shv) : nullptr;
  KernelFn fn = use_tc ? nullptr : pick(H, fp8, shv);
  size_t smem = smem_bytes(use_tc, fp8, shv, pl.tps);
  if (!ensure_smem(use_tc ? reinterpret_cast<const void*>(tfn) : reinterpret_cast<const void*>(fn),
                   static_cast<int>(smem)))
    return fail(CSA_ERR_CUDA, "%s: cannot raise the shared memory limit to %zu", name, smem);
  if (pl.cl > 1 && !use_tc) {
    static std::mutex mu;
    {
      std::lock_guard<std::mutex> lock(mu);
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        pl.cl = pl.cl > 8 ? 8 : pl.cl;  // portable cluster sizes only
      }
    }
    const int cl = choose_cluster(fn, pl.cl, R, smem, kThreads);
    if (cl != pl.cl) {  // re-plan with the co-schedulable cluster size
      const int64_t tiles = max_slots > 0 ? (max_slots + tile_keys - 1) / tile_keys : 1;
      pl.tps = static_cast<int>((tiles + cl - 1) / cl);
      pl.cl = static_cast<int>((tiles + pl.tps - 1) / pl.tps);
      smem = smem_bytes(use_tc, fp8, shv, pl.tps);
      if (!ensure_smem(reinterpret_cast<const void*>(fn), static_cast<int>(smem)))
        return fail(CSA_ERR_CUDA, "%s: cannot raise the shared memory limit to %zu", name, smem);
    }
  }

  // prefill over a bf16 cache with many query rows: the query-blocked tcgen05
  // kernel, for dense (HCA) attention and for sparse attention with few heads
  // and short selections (the block's union of selections fits on chip)
  const int qb_rows = 256 / H;
  const bool blk_shape = !fp8 && pk == nullptr && Tq >= qb_rows && R >= 2LL * num_sms();
  const bool use_blk = blk_shape && (idx == nullptr || (H == 16 && static_cast<int64_t>(qb_rows) * k <= kQbMaxCand &&
                                                        N <= kQbMaxEnt));
  CUtensorMap qmap;  // the query-blocked kernel's queries: [B][Tq*H][192] bf16, 128 x 64 boxes
  memset(&qmap, 0, sizeof(qmap));
  if (use_blk) {
    CSA_REQUIRE(Tq * H < (int64_t(1) << 31) && B < (int64_t(1) << 31), "%s: too many query rows", name);
    CSA_REQUIRE(aligned16(q), "%s: q must be 16-byte aligned", name);
    const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (encode == nullptr) return fail(CSA_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", name);
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDQK), static_cast<cuuint64_t>(Tq * H),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDQK) * 2, static_cast<cuuint64_t>(Tq * H) * kDQK * 2};
    const cuuint32_t box[3] = {64u, 128u, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUresult r = encode(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CSA_ERR_CUDA, "%s: query tensor map encoding failed (%d)", name, int(r));
    smem = qb_layout().total;
    if (!ensure_smem(reinterpret_cast<const void*>(attn_qblock_kernel), static_cast<int>(smem)))
      return fail(CSA_ERR_CUDA, "%s: cannot raise the shared memory limit to %zu", name, smem);
    pl.cl = 1;
    part = nullptr;
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
  p.part = part;
  p.cu_tok = pk ? pk->cu_tokens : nullptr;
  p.cu_ent = pk ? pk->cu_entries : nullptr;
  p.n_seqs = pk ? pk->n_seqs : 0;
  p.ent_rows = pk ? N : B * N;
  p.qb_blocks = use_blk ? B * ((Tq + qb_rows - 1) / qb_rows) : 0;
  p.win_rows = wlen > 0 ? (pk ? pk->total_tokens : B * win->rows) : 0;

  // dense query blocks: a persistent grid of one CTA per SM; sparse blocks: one CTA each
  const int64_t blk_grid = idx == nullptr ? std::min<int64_t>(p.qb_blocks, num_sms()) : p.qb_blocks;
  const dim3 grid(static_cast<unsigned>(use_blk ? blk_grid : R * pl.cl));
  const dim3 block(use_blk ? kQbThreads : (use_tc ? kTcDecThreads : kThreads));
  const int cluster = (use_tc && !tc_cluster) || use_blk ? 1 : pl.cl;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  prof_begin(s);
  const cudaError_t e = use_blk ? launch_pdl(attn_qblock_kernel, grid, block, smem, s, 1, p, qmap)
                                : launch_pdl(use_tc ? tfn : fn, grid, block, smem, s, cluster, p);
  prof_end(s);
  if (csa_status st = check_launch(name, e); st != CSA_OK) return st;
  if (part != nullptr)
    return check_launch(name, launch_pdl(attn_merge_kernel, dim3(static_cast<unsigned>(R * H / 8)), dim3(256), 0, s,
                                         1, static_cast<const float*>(part), pl.cl, H, p.out, lse));
  return CSA_OK;
}

}  // namespace
}  // namespace csa

extern "C" {

csa_status csa_check_device_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return csa::fail(CSA_ERR_CUDA, "csa_check_device_error: %s", cudaGetErrorString(e));
  int word = 0;
  e = cudaMemcpyFromSymbol(&word, csa::tc::g_device_error, sizeof(int));
  if (e != cudaSuccess) return csa::fail(CSA_ERR_CUDA, "csa_check_device_error: %s", cudaGetErrorString(e));
  for (int (*reader)(bool) : {csa::indexer_device_error, csa::compress_device_error, csa::out_proj_device_error,
                               csa::cp_merge_device_error}) {
    const int uword = reader(true);
    if (uword < 0) return csa::fail(CSA_ERR_CUDA, "csa_check_device_error: cannot read a unit's error word");
    word |= uword;
  }
  if (word != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(csa::tc::g_device_error, &zero, sizeof(int));
    return csa::fail(CSA_ERR_DEVICE_TIMEOUT, "a kernel gave up waiting on a barrier, or skipped work it could "
                     "not do in bounds (code bits %d: 1 = a bounded wait ran out, 2 = a row longer than the row "
                     "path holds, 4 = a checked build found an access out of bounds); its outputs are not valid",
                     word);
  }
  return CSA_OK;
}

csa_status csa_debug_expire_wait(void* stream) {
  csa::clear_error();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return csa::check_launch("csa_debug_expire_wait",
                           csa::launch_pdl(csa::wait_expire_kernel, dim3(1), dim3(32), 0, s, 1, uint32_t(1) << 14));
}

size_t csa_sparse_mqa_workspace_size(int64_t B, int64_t Tq, int32_t H, int32_t k, int32_t win_len) {
  if (B <= 0 || Tq <= 0 || k < 0 || win_len < 0 || B >= (1LL << 31) || Tq >= (1LL << 31) ||
      B > ((1LL << 31) - 1) / Tq)
    return 0;
  return csa::tc_part_bytes(B * Tq, H, static_cast<int64_t>(k) + win_len);
}

size_t hca_dense_mqa_workspace_size(int64_t B, int64_t Tq, int32_t H, int64_t N, int32_t win_len) {
  if (B <= 0 || Tq <= 0 || N < 0 || N >= (1LL << 31) || win_len < 0 || B >= (1LL << 31) || Tq >= (1LL << 31) ||
      B > ((1LL << 31) - 1) / Tq)
    return 0;
  return csa::tc_part_bytes(B * Tq, H, N + win_len);
}

csa_status csa_sparse_mqa(const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0, const csa_kv_cache* cache,
                          int32_t m, const int32_t* idx, int32_t k, const csa_window* win, float scale, void* out,
                          float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (idx == nullptr && B * Tq > 0)
    return csa::fail(CSA_ERR_INVALID_ARG, "csa_sparse_mqa: idx is NULL");
  return csa::run("csa_sparse_mqa", q, B, Tq, H, q_pos0, cache, m, idx, k, win, scale, out, lse, workspace,
                  workspace_bytes, stream);
}

csa_status csa_sparse_mqa_packed(const void* q, int32_t H, const csa_packed* packed, const csa_kv_cache* cache,
                                 int32_t m, const int32_t* idx, int32_t k, const csa_window* win, float scale,
                                 void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (packed == nullptr) return csa::fail(CSA_ERR_INVALID_ARG, "csa_sparse_mqa_packed: packed is NULL");
  if (idx == nullptr && packed->total_tokens > 0)
    return csa::fail(CSA_ERR_INVALID_ARG, "csa_sparse_mqa_packed: idx is NULL");
  return csa::run("csa_sparse_mqa_packed", q, 1, packed->total_tokens, H, 0, cache, m, idx, k, win, scale, out, lse,
                  workspace, workspace_bytes, stream, packed);
}

csa_status hca_dense_mqa_packed(const void* q, int32_t H, const csa_packed* packed, const csa_kv_cache* cache,
                                int32_t m_prime, const csa_window* win, float scale, void* out, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (packed == nullptr) return csa::fail(CSA_ERR_INVALID_ARG, "hca_dense_mqa_packed: packed is NULL");
  return csa::run("hca_dense_mqa_packed", q, 1, packed->total_tokens, H, 0, cache, m_prime, nullptr, 0, win, scale,
                  out, lse, workspace, workspace_bytes, stream, packed);
}

csa_status hca_dense_mqa(const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0, const csa_kv_cache* cache,
                         int32_t m_prime, const csa_window* win, float scale, void* out, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return csa::run("hca_dense_mqa", q, B, Tq, H, q_pos0, cache, m_prime, nullptr, 0, win, scale, out, lse, workspace,
                  workspace_bytes, stream);
}

csa_status hca_dense_mqa_budget(const void* q, int64_t B, int64_t Tq, int32_t H, int64_t q_pos0,
                                const csa_kv_cache* cache, int32_t m_prime, const csa_window* win, float scale,
                                void* out, float* lse, int32_t max_sms, void* workspace, size_t workspace_bytes,
                                void* stream) {
  if (max_sms < 0) return csa::fail(CSA_ERR_INVALID_ARG, "hca_dense_mqa_budget: max_sms must be >= 0");
  return csa::run("hca_dense_mqa_budget", q, B, Tq, H, q_pos0, cache, m_prime, nullptr, 0, win, scale, out, lse,
                  workspace, workspace_bytes, stream, nullptr, max_sms);
}

}  // extern "C"
