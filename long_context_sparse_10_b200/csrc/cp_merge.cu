// Merges for context-parallel decode of one long sequence over G ranks.
//
// The compressed entries of the sequence are split into G contiguous ranges,
// rank r holding entries [lo_r, lo_{r+1}).  Each rank scores its own range and
// keeps its local top-k with their scores (csa_indexer_topk_with_scores); the
// ranks exchange these candidates (an all-gather in rank order), and every
// rank selects the global top-k from the G*k candidates (csa_cp_topk_merge).
// Each rank then attends over the selected entries it holds (and one rank over
// the sliding window), giving a partial output and its log-sum-exp; after a
// second all-gather the partials are combined (csa_cp_attn_merge).  The method
// is the one of the DeepSeek-V4 summary's CSA paragraph (indexer top-k, MQA);
// splitting it over ranks this way gives exactly the single-GPU result up to
// rounding, because the global top-k is the top-k of the local top-k's and one
// softmax over disjoint key sets equals the log-sum-exp weighted merge of the
// per-set softmaxes.
#include "common.cuh"
#include "host_util.h"

namespace csa {
namespace {

constexpr int kMergeThreads = 1024;
constexpr int kMaxCand = 8 * 4096;  // candidates per row held in shared memory

__device__ __forceinline__ uint32_t scan_excl(uint32_t v, uint32_t* total, uint32_t* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = sh[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    sh[lane] = w;
  }
  __syncthreads();
  const uint32_t before = warp ? sh[warp - 1] : 0u;
  *total = sh[31];
  __syncthreads();
  return before + incl - v;
}

// One CTA per query row.  Candidate c (position in the rank-ordered list) has
// score s[c] and global index i[c] (-1: none).  Positions are in ascending
// index order (each rank's list is ascending and ranks hold increasing
// ranges), so "ties to the lower index" is "ties to the lower position" and
// an ordered compaction of the chosen positions is the ascending output.
// One CTA per query row.  Candidate c (position in the rank-ordered list) has
// score s[c] and global index i[c] (-1: none).  Positions are in ascending
// index order (each rank's list is ascending and ranks hold increasing
// ranges), so "ties to the lower index" is "ties to the lower position" and
// an ordered compaction of the chosen positions is the ascending output.  The
// k-th largest key is found by a radix select in levels of 11, 11 and 10 bits
// (2048-bin shared histograms: the candidates' scores spread over far more
// first-level bins than over the key's top byte, so the atomics collide less).
__global__ void __launch_bounds__(kMergeThreads) topk_merge_kernel(const float* __restrict__ cs,
                                                                    const int32_t* __restrict__ ci, int n, int k,
                                                                    int32_t* __restrict__ idx) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint32_t keys[];  // order-preserving score key; 0 marks an empty candidate
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t scan_sh[32];
  __shared__ uint32_t dig[2];
  const int64_t row = blockIdx.x;
  const float* srow = cs + row * n;
  const int32_t* irow = ci + row * n;
  int32_t* out = idx + row * k;
  uint32_t nvalid_local = 0;
  for (int c = threadIdx.x; c < n; c += kMergeThreads) {
    const bool ok = irow[c] >= 0;
    // valid keys are >= 1: f2key maps every float (and -inf) to a key above 0x007fffff
    keys[c] = ok ? f2key(srow[c] + 0.0f) : 0u;
    nvalid_local += ok ? 1u : 0u;
  }
  uint32_t nvalid;
  scan_excl(nvalid_local, &nvalid, scan_sh);
  uint32_t prefix = 0, remaining = static_cast<uint32_t>(k);
  if (nvalid > static_cast<uint32_t>(k)) {
    for (int level = 0; level < 3; ++level) {
      const int bits = level == 2 ? 10 : 11;
      const int shift = level == 0 ? 21 : (level == 1 ? 10 : 0);
      const uint32_t nb = 1u << bits;
      for (uint32_t j = threadIdx.x; j < nb; j += kMergeThreads) hist[j] = 0;
      __syncthreads();
      for (int c = threadIdx.x; c < n; c += kMergeThreads) {
        const uint32_t key = keys[c];
        if (key != 0u && (level == 0 || (key >> (shift + bits)) == prefix))
          atomicAdd(&hist[(key >> shift) & (nb - 1u)], 1u);
      }
      __syncthreads();
      // thread t owns bins nb-1-2t and nb-2-2t (walked from the top)
      const uint32_t b0 = nb - 1u - 2u * threadIdx.x, b1 = b0 - 1u;
      const bool own = 2u * threadIdx.x < nb;
      const uint32_t c0 = own ? hist[b0] : 0u, c1 = own ? hist[b1] : 0u;
      uint32_t total;
      const uint32_t excl = scan_excl(c0 + c1, &total, scan_sh);
      if (own && excl < remaining && excl + c0 + c1 >= remaining) {
        if (excl + c0 >= remaining) {
          dig[0] = b0;
          dig[1] = excl;
        } else {
          dig[0] = b1;
          dig[1] = excl + c0;
        }
      }
      __syncthreads();
      prefix = (prefix << bits) | dig[0];
      remaining -= dig[1];
      __syncthreads();
    }
  } else {
    prefix = 1u;  // every valid candidate (key >= 1) is above or at the threshold ...
    remaining = 0xffffffffu;  // ... and ties at it are all taken
  }
  // ordered compaction: keys above the threshold, then the first `remaining` ties
  uint32_t ties_before = 0, sel_before = 0;
  for (int base = 0; base < n; base += kMergeThreads) {
    const int c = base + threadIdx.x;
    const uint32_t key = c < n ? keys[c] : 0u;
    const bool gt = key != 0u && key > prefix;
    const bool eq = key != 0u && key == prefix;
    uint32_t tie_total;
    const uint32_t tie_rank = ties_before + scan_excl(eq ? 1u : 0u, &tie_total, scan_sh);
    const bool sel = gt || (eq && tie_rank < remaining);
    uint32_t sel_total;
    const uint32_t pos = sel_before + scan_excl(sel ? 1u : 0u, &sel_total, scan_sh);
    if (sel && pos < static_cast<uint32_t>(k)) out[pos] = irow[c];
    ties_before += tie_total;
    sel_before += sel_total;
  }
  for (uint32_t j = sel_before + threadIdx.x; j < static_cast<uint32_t>(k); j += kMergeThreads) out[j] = -1;
}

// One warp per (row, head): out = sum_g w_g o_g / sum_g w_g with
// w_g = exp(lse_g - max_g lse_g); lse = max + ln sum_g w_g.
__global__ void __launch_bounds__(256) attn_partial_merge_kernel(const __nv_bfloat16* __restrict__ outs,
                                                                 const float* __restrict__ lses, int G, int64_t RH,
                                                                 __nv_bfloat16* __restrict__ out,
                                                                 float* __restrict__ lse) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t rh = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (rh >= RH) return;
  float M = -INFINITY;
  for (int g = 0; g < G; ++g) M = fmaxf(M, __ldg(lses + g * RH + rh));
  const float base = M == -INFINITY ? 0.f : M;
  float wsum = 0.f, a[4] = {0.f, 0.f, 0.f, 0.f};
  for (int g = 0; g < G; ++g) {
    const float lg = __ldg(lses + g * RH + rh);
    const float w = lg == -INFINITY ? 0.f : __expf(lg - base);
    wsum += w;
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(outs + (g * RH + rh) * kDV) + lane);
    a[0] += w * bf16_lo(v.x);
    a[1] += w * bf16_hi(v.x);
    a[2] += w * bf16_lo(v.y);
    a[3] += w * bf16_hi(v.y);
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  reinterpret_cast<uint2*>(out + rh * kDV)[lane] =
      make_uint2(pack_bf16x2(a[0] * inv, a[1] * inv), pack_bf16x2(a[2] * inv, a[3] * inv));
  if (lane == 0 && lse != nullptr) lse[rh] = wsum > 0.f ? M + logf(wsum) : -INFINITY;
}

}  // namespace
}  // namespace csa

namespace csa {
// Reads (and optionally clears) this unit's device error word.
CSA_DEFINE_DEVICE_ERROR_READER(cp_merge_device_error)
}  // namespace csa

extern "C" {

csa_status csa_cp_topk_merge(const float* cand_scores, const int32_t* cand_idx, int64_t R, int32_t n_cand, int32_t k,
                             int32_t* idx, void* stream) {
  using namespace csa;
  clear_error();
  CSA_REQUIRE(R >= 0 && R < (int64_t(1) << 31), "csa_cp_topk_merge: R must be in [0, 2^31)");
  CSA_REQUIRE(k >= 1 && k <= 4096, "csa_cp_topk_merge: k must be in [1, 4096]");
  CSA_REQUIRE(n_cand >= 1 && n_cand <= kMaxCand, "csa_cp_topk_merge: n_cand must be in [1, %d]", kMaxCand);
  if (R == 0) return CSA_OK;
  CSA_REQUIRE(cand_scores != nullptr && (reinterpret_cast<uintptr_t>(cand_scores) & 3u) == 0,
              "csa_cp_topk_merge: cand_scores NULL or misaligned");
  CSA_REQUIRE(cand_idx != nullptr && (reinterpret_cast<uintptr_t>(cand_idx) & 3u) == 0,
              "csa_cp_topk_merge: cand_idx NULL or misaligned");
  CSA_REQUIRE(idx != nullptr && (reinterpret_cast<uintptr_t>(idx) & 3u) == 0, "csa_cp_topk_merge: idx NULL or misaligned");
  const int smem = n_cand * 4;
  if (!ensure_smem(reinterpret_cast<const void*>(topk_merge_kernel), kMaxCand * 4))
    return fail(CSA_ERR_CUDA, "csa_cp_topk_merge: cannot raise the shared memory limit");
  return check_launch("csa_cp_topk_merge",
                      launch_pdl(topk_merge_kernel, dim3(static_cast<unsigned>(R)), dim3(kMergeThreads), smem,
                                 static_cast<cudaStream_t>(stream), 1, cand_scores, cand_idx, n_cand, k, idx));
}

csa_status csa_cp_attn_merge(const void* outs, const float* lses, int32_t G, int64_t R, int32_t H, void* out,
                             float* lse, void* stream) {
  using namespace csa;
  clear_error();
  CSA_REQUIRE(G >= 1 && G <= 1024, "csa_cp_attn_merge: G must be in [1, 1024]");
  CSA_REQUIRE(R >= 0 && H >= 1 && R < (int64_t(1) << 31) / (H * G), "csa_cp_attn_merge: bad R or H");
  if (R == 0) return CSA_OK;
  CSA_REQUIRE_PTR(outs);
  CSA_REQUIRE_PTR(out);
  CSA_REQUIRE(lses != nullptr && (reinterpret_cast<uintptr_t>(lses) & 3u) == 0, "csa_cp_attn_merge: lses NULL or misaligned");
  CSA_REQUIRE(lse == nullptr || (reinterpret_cast<uintptr_t>(lse) & 3u) == 0, "csa_cp_attn_merge: lse misaligned");
  const int64_t RH = R * H;
  return check_launch("csa_cp_attn_merge",
                      launch_pdl(attn_partial_merge_kernel, dim3(static_cast<unsigned>((RH + 7) / 8)), dim3(256), 0,
                                 static_cast<cudaStream_t>(stream), 1, static_cast<const __nv_bfloat16*>(outs), lses,
                                 G, RH, static_cast<__nv_bfloat16*>(out), lse));
}

}  // extern "C"
