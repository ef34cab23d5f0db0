// Lightning indexer and top-k selection for CSA.
//
// DeepSeek-V4 paper summary (hyper.ai), section "Method", CSA paragraph: a
// "lightning indexer" scores the compressed entries and the top-k of them go
// to the core attention.  Score of entry i for query row r at position t:
//   s[r, i] = sum_{h<4} relu(qI[r,h] . kIc[i]) * wI[r,h]     (visible i: (i+1)m-1 <= t)
// and the selection keeps the k largest, ties to the lower index, returned as
// an ascending list (-1 padded when fewer than k entries are visible).
//
// Scoring is a skinny GEMM (entries x (rows*4 heads) x 64) that streams kIc
// from HBM: 16-byte cp.async copies into a 128-byte XOR-swizzled shared tile
// (4-stage pipeline), ldmatrix + bf16 tensor-core MMA (fp32 accumulate), and
// the relu/weight reduction over the 4 heads in registers.  Selection is an
// exact radix select on an order-preserving key of the fp32 score extended by
// the inverted entry index, so ties resolve to the lower index by construction:
//   * rows whose visible prefix fits in shared memory (prefill) run one CTA
//     per row over the row held in shared memory;
//   * long rows (decode over 10^5..10^6 entries) get a 4096-bin histogram of
//     the key's top 12 bits fused into the scoring kernel, whose last CTA per
//     row derives the threshold bin; one select kernel then emits a bitmap of
//     the entries above that bin plus a candidate list of the bin itself, and
//     its last CTA per row resolves the candidates and writes the ascending
//     list.  "Last CTA" is decided by an atomic counter (no CTA ever waits).
#include <mutex>

#include "common.cuh"
#include "host_util.h"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int kMaxK = 4096;
constexpr int kRowPathMaxN = 32768;  // rows up to this many visible entries live in shared memory
constexpr int kHistBins = 4096;      // first-level bins: top 12 bits of the key
constexpr int kStages = 4;
constexpr int kTileRows = 64;        // entries per pipeline stage (8 KB)
constexpr int kScoreThreads = 128;

struct ScoreParams {
  const __nv_bfloat16* qI;  // [B, Tq, 4, 64]
  const float* wI;          // [B, Tq, 4]
  const __nv_bfloat16* kI;  // [B, N, 64]
  int64_t Tq, N, q_pos0;
  int m;
  int chunk;        // entries per CTA (multiple of kTileRows)
  float* scores;    // [R, N]
  uint32_t* hist;   // [R, kHistBins] (QR == 1 only)
  uint32_t* done;   // [R, 2] CTA counters (QR == 1 only)
  int32_t* thr;     // [R, 2] threshold (QR == 1 only)
  int k;
};

__device__ __forceinline__ int64_t visible(int64_t t, int m, int64_t N) {
  int64_t v = (t + 1) / m;
  return v < N ? v : N;
}

// ---------------------------------------------------------------------------
// block-wide helpers (blockDim.x == 1024)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* total, uint32_t* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < nw ? sh[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    sh[lane] = w;
  }
  __syncthreads();
  const uint32_t before = warp ? sh[warp - 1] : 0u;
  *total = sh[nw - 1];
  __syncthreads();
  return before + incl - v;
}

// Warp 0 walks 256 bins from the top and finds the digit holding the
// `remaining`-th largest element.  Writes digit, count strictly above, and the
// bin's own count to out[0..2].
__device__ __forceinline__ void find_digit_256(const uint32_t* hist, uint32_t remaining, uint32_t* out) {
  const int lane = threadIdx.x & 31;
  uint32_t c[8], sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    c[j] = hist[255 - 8 * lane - j];
    sum += c[j];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  const uint32_t excl = incl - sum;
  if (excl < remaining && incl >= remaining) {
    uint32_t acc = excl;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (acc + c[j] >= remaining) {
        out[0] = 255 - 8 * lane - j;
        out[1] = acc;
        out[2] = c[j];
        break;
      }
      acc += c[j];
    }
  }
}

__device__ __forceinline__ void write_prefix_ids(int32_t* out, int64_t nv, int k) {
  for (int j = threadIdx.x; j < k; j += blockDim.x) out[j] = j < nv ? j : -1;
}

// Threshold of one row from its global histogram, by one CTA of NT threads
// (each owns 4096/NT consecutive bins, read as 16-byte vectors).  thr = (bin,
// count still needed from that bin); bin -1 when every visible entry fits.
template <int NT>
__device__ void row_threshold(const uint32_t* gh, int64_t nv, int k, int32_t* thr, uint32_t* scan_sh) {
  constexpr int PER = kHistBins / NT;
  static_assert(PER % 4 == 0, "bins per thread must be a multiple of 4");
  if (nv <= k) {
    if (threadIdx.x == 0) {
      thr[0] = -1;
      thr[1] = 0;
    }
    return;
  }
  // thread t owns bins [4096 - PER(t+1), 4096 - PER t), walked from the top
  const int lo = kHistBins - PER * (threadIdx.x + 1);
  uint32_t c[PER];
#pragma unroll
  for (int j = 0; j < PER / 4; ++j) {
    const uint4 v = __ldcg(reinterpret_cast<const uint4*>(gh + lo) + j);
    c[4 * j] = v.x;
    c[4 * j + 1] = v.y;
    c[4 * j + 2] = v.z;
    c[4 * j + 3] = v.w;
  }
  uint32_t sum = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) sum += c[j];
  uint32_t total;
  const uint32_t excl = block_excl_scan(sum, &total, scan_sh);
  const uint32_t kk = static_cast<uint32_t>(k);
  if (excl < kk && excl + sum >= kk) {
    uint32_t acc = excl;
#pragma unroll
    for (int j = PER - 1; j >= 0; --j) {
      if (acc + c[j] >= kk) {
        thr[0] = lo + j;
        thr[1] = static_cast<int32_t>(kk - acc);
        break;
      }
      acc += c[j];
    }
  }
}

// Scores QR consecutive query rows of one sequence against one chunk of entries.
template <int QR, bool HIST>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(ScoreParams p) {
  constexpr int NCOL = QR * 4;
  constexpr int NT = (NCOL + 7) / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* tiles = smem;
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + kStages * kTileRows * 128);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t groups = (p.Tq + QR - 1) / QR;
  const int64_t b = blockIdx.y / groups;
  const int64_t r0 = (blockIdx.y % groups) * QR;
  const int nrows = static_cast<int>((p.Tq - r0) < QR ? (p.Tq - r0) : QR);
  const int64_t nv_max = visible(p.q_pos0 + r0 + nrows - 1, p.m, p.N);
  const int64_t e_begin = static_cast<int64_t>(blockIdx.x) * p.chunk;
  if (e_begin >= nv_max) return;  // uniform for the CTA
  const int64_t e_end = (e_begin + p.chunk) < nv_max ? (e_begin + p.chunk) : nv_max;

  if (HIST) {
    for (int j = threadIdx.x; j < kHistBins; j += kScoreThreads) hist_s[j] = 0;
  }

  // B operand (k = dim, n = row*4 + head), held in registers for the whole CTA.
  uint32_t bq[4][NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int n = nt * 8 + (lane >> 2);
    const int rr = n >> 2, h = n & 3;
    const bool ok = n < NCOL && rr < nrows;
    const __nv_bfloat16* qp = p.qI + (((b * p.Tq + r0 + (ok ? rr : 0)) * kHI + h) * kDI) + (lane & 3) * 2;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      bq[kk][nt][0] = ok ? *reinterpret_cast<const uint32_t*>(qp + kk * 16) : 0u;
      bq[kk][nt][1] = ok ? *reinterpret_cast<const uint32_t*>(qp + kk * 16 + 8) : 0u;
    }
  }
  // This lane's accumulator columns: row rr = nt*2 + ((lane&3)>>1), heads (lane&1)*2 + {0,1}.
  float wv[NT][2];
  int64_t nv_r[NT];
  int64_t srow[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int rr = nt * 2 + ((lane & 3) >> 1);
    const bool ok = rr < nrows && nt * 8 < NCOL && (rr * 4) < NCOL;
    const int64_t row = b * p.Tq + r0 + (ok ? rr : 0);
    const int h0 = (lane & 1) * 2;
    wv[nt][0] = ok ? p.wI[row * kHI + h0] : 0.f;
    wv[nt][1] = ok ? p.wI[row * kHI + h0 + 1] : 0.f;
    nv_r[nt] = ok ? visible(p.q_pos0 + r0 + rr, p.m, p.N) : 0;
    srow[nt] = row;
  }

  const int ntiles = static_cast<int>((e_end - e_begin + kTileRows - 1) / kTileRows);
  const __nv_bfloat16* kbase = p.kI + b * p.N * kDI;
  auto load_tile = [&](int tile, int stage) {
    const int64_t base = e_begin + static_cast<int64_t>(tile) * kTileRows;
#pragma unroll
    for (int u = 0; u < (kTileRows * 8) / kScoreThreads; ++u) {
      const int piece = threadIdx.x + u * kScoreThreads;
      const int row = piece >> 3, ch = piece & 7;
      const int64_t e = base + row;
      const bool ok = e < e_end;
      const __nv_bfloat16* src = kbase + (ok ? e : e_begin) * kDI + ch * 8;
      uint8_t* dst = tiles + stage * (kTileRows * 128) + row * 128 + ((ch ^ (row & 7)) << 4);
      cp_async16(dst, src, ok ? 16 : 0);
    }
  };

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < ntiles) load_tile(s, s);
    cp_async_commit();
  }
  for (int tile = 0; tile < ntiles; ++tile) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    {
      const int nxt = tile + kStages - 1;
      if (nxt < ntiles) load_tile(nxt, nxt % kStages);
      cp_async_commit();
    }
    const uint8_t* st = tiles + (tile % kStages) * (kTileRows * 128);
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int ch = kk * 2 + (lane >> 4);
      uint32_t a0, a1, a2, a3;
      ldsm_x4(a0, a1, a2, a3, st + row * 128 + ((ch ^ (row & 7)) << 4));
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt], a0, a1, a2, a3, bq[kk][nt][0], bq[kk][nt][1]);
    }
    const int64_t ebase = e_begin + static_cast<int64_t>(tile) * kTileRows + warp * 16 + (lane >> 2);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float part = fmaxf(acc[nt][2 * hf], 0.f) * wv[nt][0] + fmaxf(acc[nt][2 * hf + 1], 0.f) * wv[nt][1];
        const float full = part + __shfl_xor_sync(0xffffffffu, part, 1) + 0.0f;
        const int64_t e = ebase + hf * 8;
        if ((lane & 1) == 0 && e < nv_r[nt]) {
          p.scores[srow[nt] * p.N + e] = full;
          if (HIST) atomicAdd(&hist_s[f2key(full) >> 20], 1u);
        }
      }
    }
  }
  cp_async_wait<0>();
  if (HIST) {
    // flush the CTA histogram; the row's last CTA then derives its threshold
    __shared__ uint32_t last_s;
    __shared__ uint32_t scan_sh[32];
    __syncthreads();
    const int64_t row = b * p.Tq + r0;
    uint32_t* gh = p.hist + row * kHistBins;
    for (int j = threadIdx.x; j < kHistBins; j += kScoreThreads) {
      const uint32_t c = hist_s[j];
      if (c) atomicAdd(gh + j, c);
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const uint32_t ctas = static_cast<uint32_t>((nv_max + p.chunk - 1) / p.chunk);
      last_s = (atomicAdd(p.done + 2 * row, 1u) == ctas - 1) ? 1u : 0u;
    }
    __syncthreads();
    if (last_s) {
      __threadfence();
      row_threshold<kScoreThreads>(gh, nv_max, p.k, p.thr + 2 * row, scan_sh);
    }
  }
}

// ---------------------------------------------------------------------------
// row path: one CTA (1024 threads) per query row, row held in shared memory
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) topk_rows_kernel(const float* __restrict__ scores, int64_t N, int64_t Tq,
                                                         int64_t q_pos0, int m, int k, int32_t* __restrict__ idx) {
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t dig[3];
  __shared__ uint32_t scan_sh[32];
  const int64_t row = blockIdx.x;
  const int64_t nv = visible(q_pos0 + row % Tq, m, N);
  int32_t* out = idx + row * k;
  if (nv <= k) {
    write_prefix_ids(out, nv, k);
    return;
  }
  const float* srow = scores + row * N;
  for (int64_t i = threadIdx.x; i < nv; i += blockDim.x) keys[i] = f2key(srow[i]);
  uint32_t prefix = 0, mask = 0, remaining = static_cast<uint32_t>(k);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int j = threadIdx.x; j < 256; j += blockDim.x) hist[j] = 0;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < nv; i += blockDim.x) {
      const uint32_t key = keys[i];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) find_digit_256(hist, remaining, dig);
    __syncthreads();
    prefix |= dig[0] << shift;
    mask |= 255u << shift;
    remaining -= dig[1];
    __syncthreads();
  }
  // kth key = prefix; all keys > prefix plus the `remaining` lowest-index keys == prefix.
  uint32_t ties_before = 0, sel_before = 0;
  for (int64_t base = 0; base < nv; base += blockDim.x) {
    const int64_t i = base + threadIdx.x;
    const uint32_t key = i < nv ? keys[i] : 0u;
    const bool gt = i < nv && key > prefix;
    const bool eq = i < nv && key == prefix;
    uint32_t tie_total;
    const uint32_t tie_rank = ties_before + block_excl_scan(eq ? 1u : 0u, &tie_total, scan_sh);
    const bool sel = gt || (eq && tie_rank < remaining);
    uint32_t sel_total;
    const uint32_t pos = sel_before + block_excl_scan(sel ? 1u : 0u, &sel_total, scan_sh);
    if (sel) out[pos] = static_cast<int32_t>(i);
    ties_before += tie_total;
    sel_before += sel_total;
  }
}

// ---------------------------------------------------------------------------
// long-row path: histogram + threshold fused into scoring, then one select
// kernel whose last CTA per row resolves the threshold bin and writes the list
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 512;
constexpr int kSelChunk = 8192;         // entries per select CTA
constexpr int kCandSmem = 4096;         // threshold-bin candidates kept in shared memory
constexpr int kBitmapSmemWords = 8192;  // rows up to 262144 entries emit from a shared-memory bitmap

struct LongWs {
  float* scores;        // [R, N]
  uint32_t* hist;       // [R, kHistBins]    (zeroed per call)
  uint32_t* cand_cnt;   // [R]               (zeroed per call)
  uint32_t* done;       // [R, 2]: scoring / select CTAs finished (zeroed per call)
  int32_t* thr;         // [R, 2]
  uint2* cand;          // [R, N]: (key, index) of the threshold bin's entries
  uint32_t* bitmap;     // [R, W]
  int64_t W;
};

// Per CTA: a bitmap word for every 32 entries (entries above the threshold
// bin), and the threshold bin's entries appended to the row's candidate list
// (gathered in shared memory first, one global atomic per CTA).  The last CTA
// of a row then radix-selects the `need` best candidates on the composite key
// (score key << 32 | ~index), merges them into the row's bitmap and writes the
// ascending index list.  Rows up to kBitmapSmemWords*32 entries keep that final
// bitmap in shared memory.
__global__ void __launch_bounds__(kSelThreads, 2) topk_select_kernel(LongWs ws, int64_t N, int64_t Tq, int64_t q_pos0,
                                                                     int m, int k, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t sel_smem[];  // candidates, then the final bitmap
  uint2* cand_s = reinterpret_cast<uint2*>(sel_smem);
  uint32_t* bm_s = reinterpret_cast<uint32_t*>(sel_smem + kCandSmem * sizeof(uint2));
  __shared__ uint32_t hist[256];
  __shared__ uint32_t dig[3];
  __shared__ uint32_t scan_sh[32];
  __shared__ uint32_t n_cand, base_s, last_s, spill_base;
  const int64_t row = blockIdx.y;
  const int64_t nv = visible(q_pos0 + row % Tq, m, N);
  const int64_t e_begin = static_cast<int64_t>(blockIdx.x) * kSelChunk;
  if (e_begin >= nv) return;
  int32_t* out = idx + row * k;
  const int thr_bin = ws.thr[2 * row];
  if (thr_bin < 0) {  // every visible entry is selected
    if (blockIdx.x == 0) write_prefix_ids(out, nv, k);
    return;
  }
  const int64_t e_end = (e_begin + kSelChunk) < nv ? (e_begin + kSelChunk) : nv;
  const uint32_t tb = static_cast<uint32_t>(thr_bin);
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) n_cand = 0;
  __syncthreads();
  const float* srow = ws.scores + row * N;
  constexpr int kIters = kSelChunk / kSelThreads;
  float sv[kIters];
#pragma unroll
  for (int it = 0; it < kIters; ++it) {  // all loads first, then the bookkeeping
    const int64_t i = e_begin + it * kSelThreads + threadIdx.x;
    sv[it] = i < e_end ? __ldcg(srow + i) : 0.f;
  }
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int64_t base = e_begin + it * kSelThreads + (threadIdx.x & ~31);
    const int64_t i = base + lane;
    const bool ok = i < e_end;
    const uint32_t key = ok ? f2key(sv[it]) : 0u;
    const uint32_t bin = key >> 20;
    const uint32_t word = __ballot_sync(0xffffffffu, ok && bin > tb);
    if (lane == 0 && base < e_end) ws.bitmap[row * ws.W + (base >> 5)] = word;
    const bool cnd = ok && bin == tb;
    const uint32_t cm = __ballot_sync(0xffffffffu, cnd);
    if (cm) {
      uint32_t pos = 0;
      if (lane == 0) pos = atomicAdd(&n_cand, static_cast<uint32_t>(__popc(cm)));
      pos = __shfl_sync(0xffffffffu, pos, 0);
      const uint32_t my = pos + __popc(cm & ((1u << lane) - 1u));
      if (cnd) {
        if (my < static_cast<uint32_t>(kCandSmem)) {
          cand_s[my] = make_uint2(key, static_cast<uint32_t>(i));
        } else {  // rare (many equal scores): straight to the row's list
          ws.cand[row * N + atomicAdd(ws.cand_cnt + row, 1u)] = make_uint2(key, static_cast<uint32_t>(i));
        }
      }
    }
  }
  __syncthreads();
  const uint32_t nc = n_cand < static_cast<uint32_t>(kCandSmem) ? n_cand : static_cast<uint32_t>(kCandSmem);
  if (threadIdx.x == 0 && nc) base_s = atomicAdd(ws.cand_cnt + row, nc);
  __syncthreads();
  for (uint32_t c = threadIdx.x; c < nc; c += kSelThreads) ws.cand[row * N + base_s + c] = cand_s[c];
  // last CTA of this row?
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t chunks = static_cast<uint32_t>((nv + kSelChunk - 1) / kSelChunk);
    last_s = (atomicAdd(ws.done + 2 * row + 1, 1u) == chunks - 1) ? 1u : 0u;
  }
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  (void)spill_base;

  // ---- load the row's candidates (when they fit) and bitmap (when it fits) together
  const int64_t words = (nv + 31) >> 5;
  const uint32_t cnt = __ldcg(ws.cand_cnt + row);
  const uint2* cand = ws.cand + row * N;
  uint32_t* gbm = ws.bitmap + row * ws.W;
  const bool bm_in_smem = words <= kBitmapSmemWords;
  const bool cand_in_smem = cnt <= static_cast<uint32_t>(kCandSmem);
  if (bm_in_smem) {
    for (int64_t w0 = 4 * threadIdx.x; w0 < words; w0 += 4 * kSelThreads) {
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(gbm + w0));
      bm_s[w0] = v.x;
      if (w0 + 1 < words) bm_s[w0 + 1] = v.y;
      if (w0 + 2 < words) bm_s[w0 + 2] = v.z;
      if (w0 + 3 < words) bm_s[w0 + 3] = v.w;
    }
  }
  if (cand_in_smem) {
    for (uint32_t c0 = 0; c0 < cnt; c0 += 4 * kSelThreads) {
      uint2 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t c = c0 + u * kSelThreads + threadIdx.x;
        v[u] = c < cnt ? __ldcg(cand + c) : make_uint2(0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t c = c0 + u * kSelThreads + threadIdx.x;
        if (c < cnt) cand_s[c] = v[u];
      }
    }
    cand = cand_s;
  }
  __syncthreads();

  // ---- resolve the threshold bin: radix select on the 52 low composite bits
  uint32_t remaining = static_cast<uint32_t>(ws.thr[2 * row + 1]);
  uint64_t prefix = static_cast<uint64_t>(thr_bin) << 52;
  uint64_t mask = 0xfffull << 52;
  uint32_t in_bucket = cnt;
  for (int pass = 0; pass < 7 && in_bucket != remaining; ++pass) {
    const int sh = pass < 6 ? 44 - 8 * pass : 0;
    const uint64_t dmask = pass < 6 ? 255ull : 15ull;
    for (int j = threadIdx.x; j < 256; j += kSelThreads) hist[j] = 0;
    __syncthreads();
    for (uint32_t c = threadIdx.x; c < cnt; c += kSelThreads) {
      const uint2 kv = cand_in_smem ? cand[c] : __ldcg(cand + c);
      const uint64_t x = (static_cast<uint64_t>(kv.x) << 32) | (0xffffffffu - kv.y);
      if ((x & mask) == prefix) atomicAdd(&hist[(x >> sh) & dmask], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) find_digit_256(hist, remaining, dig);
    __syncthreads();
    prefix |= static_cast<uint64_t>(dig[0]) << sh;
    mask |= dmask << sh;
    remaining -= dig[1];
    in_bucket = dig[2];
    __syncthreads();
  }
  uint32_t* bm = bm_in_smem ? bm_s : gbm;
  for (uint32_t c = threadIdx.x; c < cnt; c += kSelThreads) {
    const uint2 kv = cand_in_smem ? cand[c] : __ldcg(cand + c);
    const uint64_t x = (static_cast<uint64_t>(kv.x) << 32) | (0xffffffffu - kv.y);
    if ((x & mask) >= prefix) atomicOr(bm + (kv.y >> 5), 1u << (kv.y & 31));
  }
  if (!bm_in_smem) __threadfence();
  __syncthreads();

  // ---- ascending list from the bitmap: 16 consecutive words per thread per round
  uint32_t before = 0;
  for (int64_t base = 0; base < words; base += 16 * kSelThreads) {
    const int64_t w0 = base + 16 * threadIdx.x;
    uint32_t wv[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int64_t wi = w0 + j;
      uint32_t word = 0;
      if (wi < words) word = bm_in_smem ? bm_s[wi] : __ldcg(gbm + wi);
      if (wi == words - 1 && (nv & 31)) word &= (1u << (nv & 31)) - 1u;
      wv[j] = word;
    }
    uint32_t cntw = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) cntw += __popc(wv[j]);
    uint32_t total;
    uint32_t pos = before + block_excl_scan(cntw, &total, scan_sh);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      uint32_t word = wv[j];
      while (word) {
        const int bit = __ffs(word) - 1;
        word &= word - 1;
        if (pos < static_cast<uint32_t>(k)) out[pos] = static_cast<int32_t>(((w0 + j) << 5) + bit);
        ++pos;
      }
    }
    before += total;
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool use_row_path(int64_t R, int64_t N) { return N <= kRowPathMaxN && R > 256; }

struct LongLayout {
  size_t scores, hist, cnt, done, thr, cand, bitmap, total;
  int64_t W;
};

LongLayout long_layout(int64_t R, int64_t N) {
  LongLayout L;
  L.W = ((N + 31) / 32 + 15) / 16 * 16;  // 16-word multiple: vector reads stay in the row
  size_t off = 0;
  L.scores = off; off = align_up(off + static_cast<size_t>(R) * N * 4);
  L.hist = off;   off += static_cast<size_t>(R) * kHistBins * 4;     // hist, cnt and done: zeroed together
  L.cnt = off;    off += static_cast<size_t>(R) * 4;
  L.done = off;   off = align_up(off + static_cast<size_t>(R) * 8);
  L.thr = off;    off = align_up(off + static_cast<size_t>(R) * 8);
  L.cand = off;   off = align_up(off + static_cast<size_t>(R) * N * 8);
  L.bitmap = off; off = align_up(off + static_cast<size_t>(R) * L.W * 4);
  L.total = off;
  return L;
}

size_t workspace_bytes(int64_t B, int64_t Tq, int64_t N) {
  const int64_t R = B * Tq;
  if (R <= 0 || N <= 0) return 0;
  if (use_row_path(R, N)) return align_up(static_cast<size_t>(R) * N * 4);
  return long_layout(R, N).total;
}

}  // namespace
}  // namespace csa

namespace csa {
// Reads (and optionally clears) this unit's device error word.
int indexer_device_error(bool clear) {
  int word = 0;
  if (cudaMemcpyFromSymbol(&word, tc::g_device_error, sizeof(int)) != cudaSuccess) return -1;
  if (word && clear) {
    const int zero = 0;
    cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(int));
  }
  return word;
}
}  // namespace csa

extern "C" {

size_t csa_indexer_topk_workspace_size(int64_t B, int64_t Tq, int64_t N, int32_t k) {
  (void)k;
  if (B < 0 || Tq < 0 || N < 0) return 0;
  return csa::workspace_bytes(B, Tq, N);
}

csa_status csa_indexer_topk(const void* qI, const float* wI, const void* kIc, int64_t B, int64_t Tq, int64_t N,
                            int64_t q_pos0, int32_t m, int32_t k, int32_t* idx, void* workspace,
                            size_t workspace_bytes, void* stream) {
  using namespace csa;
  clear_error();
  CSA_REQUIRE(B >= 0 && Tq >= 0 && N >= 0, "csa_indexer_topk: negative size");
  CSA_REQUIRE(N < (1LL << 31), "csa_indexer_topk: N must be < 2^31");
  CSA_REQUIRE(m >= 1, "csa_indexer_topk: m must be >= 1");
  CSA_REQUIRE(k >= 1 && k <= kMaxK, "csa_indexer_topk: k must be in [1, %d] (got %d)", kMaxK, k);
  CSA_REQUIRE(q_pos0 >= 0, "csa_indexer_topk: q_pos0 must be >= 0");
  const int64_t R = B * Tq;
  if (R == 0) return CSA_OK;
  CSA_REQUIRE(R < (1LL << 31), "csa_indexer_topk: too many query rows");
  CSA_REQUIRE_PTR(idx);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (N == 0) {
    if (cudaMemsetAsync(idx, 0xff, static_cast<size_t>(R) * k * 4, s) != cudaSuccess)
      return fail(CSA_ERR_CUDA, "csa_indexer_topk: memset failed");
    return CSA_OK;
  }
  CSA_REQUIRE_PTR(qI);
  CSA_REQUIRE_PTR(wI);
  CSA_REQUIRE_PTR(kIc);
  const size_t need = csa::workspace_bytes(B, Tq, N);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "csa_indexer_topk: workspace of %zu bytes needed (got %zu)", need,
                workspace_bytes);
  CSA_REQUIRE(aligned16(workspace), "csa_indexer_topk: workspace is not 16-byte aligned");

  ScoreParams p;
  p.qI = static_cast<const __nv_bfloat16*>(qI);
  p.wI = wI;
  p.kI = static_cast<const __nv_bfloat16*>(kIc);
  p.Tq = Tq;
  p.N = N;
  p.q_pos0 = q_pos0;
  p.m = m;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t tile_smem = static_cast<size_t>(kStages) * kTileRows * 128;

  if (use_row_path(R, N)) {
    constexpr int QR = 8;
    p.chunk = 2048;
    p.scores = reinterpret_cast<float*>(ws);
    p.hist = nullptr;
    p.done = nullptr;
    p.thr = nullptr;
    p.k = k;
    const int64_t groups = (Tq + QR - 1) / QR;
    dim3 grid(static_cast<unsigned>((N + p.chunk - 1) / p.chunk), static_cast<unsigned>(B * groups));
    CSA_REQUIRE(B * groups < 65536, "csa_indexer_topk: too many query rows for one launch");
    prof_begin(s);
    score_kernel<QR, false><<<grid, kScoreThreads, tile_smem, s>>>(p);
    prof_end(s);
    if (csa_status st = check_launch("indexer score"); st != CSA_OK) return st;
    const size_t smem = static_cast<size_t>(N) * 4;
    if (!ensure_smem(reinterpret_cast<const void*>(topk_rows_kernel), kRowPathMaxN * 4))
      return fail(CSA_ERR_CUDA, "csa_indexer_topk: cannot raise shared memory limit");
    topk_rows_kernel<<<static_cast<unsigned>(R), 1024, smem, s>>>(p.scores, N, Tq, q_pos0, m, k, idx);
    return check_launch("indexer top-k (rows)");
  }

  const LongLayout L = long_layout(R, N);
  LongWs w;
  w.scores = reinterpret_cast<float*>(ws + L.scores);
  w.hist = reinterpret_cast<uint32_t*>(ws + L.hist);
  w.cand_cnt = reinterpret_cast<uint32_t*>(ws + L.cnt);
  w.done = reinterpret_cast<uint32_t*>(ws + L.done);
  w.thr = reinterpret_cast<int32_t*>(ws + L.thr);
  w.cand = reinterpret_cast<uint2*>(ws + L.cand);
  w.bitmap = reinterpret_cast<uint32_t*>(ws + L.bitmap);
  w.W = L.W;
  if (cudaMemsetAsync(w.hist, 0, L.thr - L.hist, s) != cudaSuccess)
    return fail(CSA_ERR_CUDA, "csa_indexer_topk: memset failed");
  p.chunk = 4096;
  p.scores = w.scores;
  p.hist = w.hist;
  p.done = w.done;
  p.thr = w.thr;
  p.k = k;
  CSA_REQUIRE(R < 65536, "csa_indexer_topk: too many query rows for the long-row path");
  dim3 grid(static_cast<unsigned>((N + p.chunk - 1) / p.chunk), static_cast<unsigned>(R));
  if (!ensure_smem(reinterpret_cast<const void*>(score_kernel<1, true>), tile_smem + kHistBins * 4))
    return fail(CSA_ERR_CUDA, "csa_indexer_topk: cannot raise shared memory limit");
  prof_begin(s);
  score_kernel<1, true><<<grid, kScoreThreads, tile_smem + kHistBins * 4, s>>>(p);
  prof_end(s);
  if (csa_status st = check_launch("indexer score (long rows)"); st != CSA_OK) return st;
  dim3 sgrid(static_cast<unsigned>((N + kSelChunk - 1) / kSelChunk), static_cast<unsigned>(R));
  constexpr int kSelSmem = kCandSmem * 8 + kBitmapSmemWords * 4;
  if (!ensure_smem(reinterpret_cast<const void*>(topk_select_kernel), kSelSmem))
    return fail(CSA_ERR_CUDA, "csa_indexer_topk: cannot raise shared memory limit");
  topk_select_kernel<<<sgrid, kSelThreads, kSelSmem, s>>>(w, N, Tq, q_pos0, m, k, idx);
  return check_launch("indexer select");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// csa_indexer_topk_noalloc: the same selection with library-owned scratch.
//
// Some callers cannot allocate device memory themselves -- for example a plugin
// whose host application owns every device allocation, or code on a latency-
// critical path that must not call cudaMalloc.  This variant takes no
// workspace: it uses a file-scope static device array of
// kStaticScratchBytes (32 MiB), which every GPU that loads the library holds
// until the process exits.  Host code cannot hand the array's name to a kernel
// (on the host it is only a stand-in for the symbol), so the first call on
// each device looks up the array's device address with cudaGetSymbolAddress
// while that device is current and caches it; that first call should come
// before any stream capture.  The call itself allocates nothing: it forwards
// to csa_indexer_topk with the cached address as the workspace, and that path
// clears the parts of the scratch that must start at zero on every call.  All
// calls share the one array and it keeps the last call's contents, so calls
// that overlap on the GPU (different streams, or host threads, without
// ordering between them) race on it.
// ---------------------------------------------------------------------------
static constexpr size_t kStaticScratchBytes = static_cast<size_t>(32) << 20;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];
static std::mutex g_static_mu;
static void* g_static_ptr[64] = {nullptr};

extern "C" csa_status csa_indexer_topk_noalloc(const void* qI, const float* wI, const void* kIc, int64_t B,
                                               int64_t Tq, int64_t N, int64_t q_pos0, int32_t m, int32_t k,
                                               int32_t* idx, void* stream) {
  using namespace csa;
  if (B < 0 || Tq < 0 || N < 0) return fail(CSA_ERR_INVALID_ARG, "csa_indexer_topk_noalloc: negative size");
  const size_t need = csa::workspace_bytes(B, Tq, N);
  if (need > kStaticScratchBytes)
    return fail(CSA_ERR_UNSUPPORTED,
                "csa_indexer_topk_noalloc: these sizes need %zu bytes of scratch but the static scratch holds %zu; "
                "call csa_indexer_topk with a caller workspace instead",
                need, kStaticScratchBytes);
  void* ptr = nullptr;
  if (need > 0) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
      return fail(CSA_ERR_CUDA, "csa_indexer_topk_noalloc: no usable current device");
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_ptr[dev] == nullptr) {
      const cudaError_t e = cudaGetSymbolAddress(&g_static_ptr[dev], g_static_scratch);
      if (e != cudaSuccess) {
        g_static_ptr[dev] = nullptr;
        return fail(CSA_ERR_CUDA, "csa_indexer_topk_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
      }
    }
    ptr = g_static_ptr[dev];
  }
  return csa_indexer_topk(qI, wI, kIc, B, Tq, N, q_pos0, m, k, idx, ptr, ptr ? kStaticScratchBytes : 0, stream);
}
