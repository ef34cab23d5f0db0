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
// from HBM into 128-byte XOR-swizzled shared tiles -- by TMA with an L2
// evict-first policy for long rows (score_long_kernel), by 16-byte cp.async
// copies for prefill rows (score_kernel) -- then ldmatrix + bf16 tensor-core
// MMA (fp32 accumulate) and the relu/weight reduction over the 4 heads in
// registers; E4M3 keys are widened to fp16 in registers.  Selection is an
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
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "host_util.h"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int kMaxK = 4096;
constexpr int kRowPathMaxN = 32768;  // rows up to this many visible entries live in shared memory
constexpr int kHistBins = 4096;      // first-level bins: top 12 bits of the key
// Scoring pipeline shape (compile-time tunables): stages of kTileRows entries
// (128 B each) per CTA of kScoreThreads threads; each warp owns 16 rows of a stage.
#ifndef CSA_SCORE_STAGES
#define CSA_SCORE_STAGES 4
#endif
#ifndef CSA_SCORE_WARPS
#define CSA_SCORE_WARPS 4
#endif
constexpr int kStages = CSA_SCORE_STAGES;
constexpr int kScoreThreads = 32 * CSA_SCORE_WARPS;
constexpr int kTileRows = 16 * CSA_SCORE_WARPS;  // entries per pipeline stage

struct ScoreParams {
  const __nv_bfloat16* qI;  // [B, Tq, 4, 64]
  const float* wI;          // [B, Tq, 4]
  const __nv_bfloat16* kI;  // [B, N, 64] (bf16 keys)
  const uint8_t* kcodes;    // [B, N, 64] E4M3 key codes (E4 variant)
  const float* kscale;      // [B, N] per-entry scale (E4 variant)
  int64_t Tq, N, q_pos0;
  int m;
  int chunk;        // entries per CTA (multiple of 2 * kTileRows)
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
// Shared memory of the scoring kernel: bf16 keys: kStages swizzled tiles;
// E4M3 keys: kStages stages of codes + scales, twice the entries per stage
// (same bytes per stage); then the histogram (HIST).
__host__ __device__ constexpr size_t score_tile_bytes(bool e4) {
  return e4 ? static_cast<size_t>(kStages) * (2 * kTileRows) * (64 + 4)
            : static_cast<size_t>(kStages) * kTileRows * 128;
}

// E4M3 keys feed an fp16 MMA straight from registers.  The dot product over
// the 64 dimensions may visit them in any order as long as A (keys) and B
// (query) agree, so lane (g = lane/4, t = lane%4) takes dims 16t .. 16t+15 of
// its key rows with one 16-byte shared load: k-step j, fragment slots
// {2t, 2t+1, 2t+8, 2t+9} <- dims 16t + 4j + {0, 1, 2, 3}.  The query is scaled
// per (row, head) by a power of two 2^e that brings its largest magnitude into
// [2^14, 2^15) before the fp16 conversion (exact for every bf16 value in that
// head down to 2^-28 of its maximum), and 2^-e moves onto the head weight:
// relu(2^e x) 2^-e w = relu(x) w.
template <int QR, bool E4>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(ScoreParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr int NCOL = QR * 4;
  constexpr int NT = (NCOL + 7) / 8;
  constexpr int TR = E4 ? 2 * kTileRows : kTileRows;  // entries per stage
  constexpr int MT = TR / kTileRows;                  // 16-row MMA tiles per warp and stage
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* tiles = smem;                                             // bf16: [kStages] swizzled tiles
  uint8_t* codes_st = smem;                                          // E4: [kStages][TR][64]
  float* scale_st = reinterpret_cast<float*>(smem + kStages * TR * 64);  // E4: [kStages][TR]

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t groups = (p.Tq + QR - 1) / QR;
  const int64_t b = blockIdx.y / groups;
  const int64_t r0 = (blockIdx.y % groups) * QR;
  const int nrows = static_cast<int>((p.Tq - r0) < QR ? (p.Tq - r0) : QR);
  const int64_t nv_max = visible(p.q_pos0 + r0 + nrows - 1, p.m, p.N);
  const int64_t e_begin = static_cast<int64_t>(blockIdx.x) * p.chunk;
  if (e_begin >= nv_max) return;  // uniform for the CTA
  const int64_t e_end = (e_begin + p.chunk) < nv_max ? (e_begin + p.chunk) : nv_max;

  // B operand (k = dim, n = row*4 + head), held in registers for the whole CTA.
  uint32_t bq[4][NT][2];
  int qexp[NT];  // E4: exponent e of column n = nt*8 + lane/4
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int n = nt * 8 + (lane >> 2);
    const int rr = n >> 2, h = n & 3;
    const bool ok = n < NCOL && rr < nrows;
    const __nv_bfloat16* qrow = p.qI + (((b * p.Tq + r0 + (ok ? rr : 0)) * kHI + h) * kDI);
    if (E4) {
      const __nv_bfloat16* qp = qrow + (lane & 3) * 16;
      float qv[16];
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        qv[i] = ok ? __bfloat162float(qp[i]) : 0.f;
        amax = fmaxf(amax, fabsf(qv[i]));
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      int e = 14 - (static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127);
      e = amax > 0.f ? (e < -60 ? -60 : (e > 60 ? 60 : e)) : 0;
      qexp[nt] = e;
      const float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        bq[kk][nt][0] = pack_f16x2(qv[4 * kk] * sc, qv[4 * kk + 1] * sc);
        bq[kk][nt][1] = pack_f16x2(qv[4 * kk + 2] * sc, qv[4 * kk + 3] * sc);
      }
    } else {
      const __nv_bfloat16* qp = qrow + (lane & 3) * 2;
      qexp[nt] = 0;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        bq[kk][nt][0] = ok ? *reinterpret_cast<const uint32_t*>(qp + kk * 16) : 0u;
        bq[kk][nt][1] = ok ? *reinterpret_cast<const uint32_t*>(qp + kk * 16 + 8) : 0u;
      }
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
    if (E4) {  // columns 2t, 2t+1 of this n-tile were scaled by the lanes with g = 2t, 2t+1
      const int e0 = __shfl_sync(0xffffffffu, qexp[nt], 4 * (2 * (lane & 3)));
      const int e1 = __shfl_sync(0xffffffffu, qexp[nt], 4 * (2 * (lane & 3) + 1));
      wv[nt][0] *= __uint_as_float(static_cast<uint32_t>(127 - e0) << 23);
      wv[nt][1] *= __uint_as_float(static_cast<uint32_t>(127 - e1) << 23);
    }
    nv_r[nt] = ok ? visible(p.q_pos0 + r0 + rr, p.m, p.N) : 0;
    srow[nt] = row;
  }

  const int ntiles = static_cast<int>((e_end - e_begin + TR - 1) / TR);
  const __nv_bfloat16* kbase = p.kI + b * p.N * kDI;
  auto load_tile = [&](int tile, int stage) {
    const int64_t base = e_begin + static_cast<int64_t>(tile) * TR;
    if constexpr (E4) {
      // 64 code bytes per entry (4 pieces) and one 4-byte scale per entry
      for (int piece = threadIdx.x; piece < TR * 4; piece += kScoreThreads) {
        const int row = piece >> 2, ch = piece & 3;
        const int64_t e = base + row;
        const bool ok = e < e_end;
        cp_async16(codes_st + (stage * TR + row) * 64 + ch * 16,
                   p.kcodes + (b * p.N + (ok ? e : e_begin)) * kDI + ch * 16, ok ? 16 : 0);
      }
      for (int row = threadIdx.x; row < TR; row += kScoreThreads) {
        const int64_t e = base + row;
        if (e < e_end) {
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(scale_st + stage * TR + row)),
                       "l"(p.kscale + b * p.N + e));
        } else {
          scale_st[stage * TR + row] = 0.f;
        }
      }
    } else {
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
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int rbase = warp * (16 * MT) + mt * 16;  // this warp's first row of the stage
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      if (E4) {
        const uint8_t* cs = codes_st + ((tile % kStages) * TR + rbase + (lane >> 2)) * 64 + (lane & 3) * 16;
        const uint4 lo = *reinterpret_cast<const uint4*>(cs);
        const uint4 hi = *reinterpret_cast<const uint4*>(cs + 8 * 64);
        const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w}, wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t a0, a1, a2, a3;
          e4m3x4_to_f16x2x2(wl[kk], a0, a2);
          e4m3x4_to_f16x2x2(wh[kk], a1, a3);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_f16(acc[nt], a0, a1, a2, a3, bq[kk][nt][0], bq[kk][nt][1]);
        }
      } else {
        const uint8_t* st = tiles + (tile % kStages) * (kTileRows * 128);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int row = rbase + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int ch = kk * 2 + (lane >> 4);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(a0, a1, a2, a3, st + row * 128 + ((ch ^ (row & 7)) << 4));
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt], a0, a1, a2, a3, bq[kk][nt][0], bq[kk][nt][1]);
        }
      }
      const int64_t ebase = e_begin + static_cast<int64_t>(tile) * TR + rbase + (lane >> 2);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float part = fmaxf(acc[nt][2 * hf], 0.f) * wv[nt][0] + fmaxf(acc[nt][2 * hf + 1], 0.f) * wv[nt][1];
          float full = part + __shfl_xor_sync(0xffffffffu, part, 1);
          const int64_t e = ebase + hf * 8;
          if (E4)  // scale > 0 factors out of relu: score = scale * sum_h relu(q_h . codes) w_h
            full *= scale_st[(tile % kStages) * TR + rbase + (lane >> 2) + hf * 8];
          full += 0.0f;
          if ((lane & 1) == 0 && e < nv_r[nt]) {
            p.scores[srow[nt] * p.N + e] = full;
          }
        }
      }
    }
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// long rows: one query row per CTA row of the grid, histogram fused
// ---------------------------------------------------------------------------
// Each CTA scores one chunk of one row.  Stages of kLongTR entries arrive by
// bulk copy (bf16 keys: one TMA box of a [B][N][64] tensor map with the
// 128-byte swizzle that ldmatrix reads conflict-free; E4M3 keys: one
// contiguous copy of the codes, plus 4-byte cp.async copies of the scales),
// each completing on its stage's mbarrier.  Each warp owns 32 entries of a
// stage: two 16-row MMA tiles whose 4 useful accumulator columns (the 4
// heads) are folded so that every lane ends with one entry's score, and the
// score store and histogram update run once per entry on all 32 lanes.
constexpr int kLongThreads = 128;
constexpr int kLongTR = 128;  // entries per stage (32 per warp)
constexpr int kLongMinChunk = 1024;
constexpr int kLongMaxChunk = 65536 - kLongTR;  // per-CTA bin counts fit 16 bits

#ifndef CSA_LONG_STAGES_BF16
#define CSA_LONG_STAGES_BF16 3
#endif
#ifndef CSA_LONG_STAGES_E4
#define CSA_LONG_STAGES_E4 4
#endif
template <bool E4>
struct LongShape {
  static constexpr int kStages = E4 ? CSA_LONG_STAGES_E4 : CSA_LONG_STAGES_BF16;
  static constexpr int kStageBytes = kLongTR * (E4 ? 64 : 128);
  static constexpr size_t kScaleOff = static_cast<size_t>(kStages) * kStageBytes;
  static constexpr size_t kHistOff = kScaleOff + (E4 ? static_cast<size_t>(kStages) * kLongTR * 4 : 0);
  static constexpr size_t kBarOff = kHistOff + kHistBins * 2;  // two 16-bit bins per word
  static constexpr size_t kSmem = kBarOff + kStages * 8 + 1024;  // + alignment slack for the 1024-byte swizzle atoms
};

struct LongScoreParams {
  const __nv_bfloat16* qI;  // [B, Tq, 4, 64]
  const float* wI;          // [B, Tq, 4]
  const uint8_t* kcodes;    // [B, N, 64] (E4)
  const float* kscale;      // [B, N] (E4)
  int64_t Tq, N, q_pos0;
  int m;
  int chunk;  // entries per CTA, a multiple of kLongTR
  int64_t pitch;  // row pitch of scores
  float* scores;
  uint32_t* hist;
  uint32_t* done;
  int32_t* thr;
  int k;
};

template <bool E4>
__global__ void __launch_bounds__(kLongThreads) score_long_kernel(LongScoreParams p,
                                                                  const __grid_constant__ CUtensorMap kmap) {
  pdl_wait();
  using S = LongShape<E4>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float* scale_st = reinterpret_cast<float*>(smem + S::kScaleOff);  // E4: [kStages][kLongTR]
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + S::kHistOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  __shared__ uint32_t last_s;
  __shared__ uint32_t scan_sh[32];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int64_t row = blockIdx.y;
  const int64_t b = row / p.Tq;
  const int64_t nv = visible(p.q_pos0 + row % p.Tq, p.m, p.N);
  const int64_t e_begin = static_cast<int64_t>(blockIdx.x) * p.chunk;
  if (e_begin >= nv) return;  // uniform for the CTA
  const int64_t e_end = (e_begin + p.chunk) < nv ? (e_begin + p.chunk) : nv;
  const int ntiles = static_cast<int>((e_end - e_begin + kLongTR - 1) / kLongTR);

  for (int j = threadIdx.x; j < kHistBins / 2; j += kLongThreads) hist_s[j] = 0;
  if (threadIdx.x == 0) {
    for (int st = 0; st < S::kStages; ++st) tc::bar_init(&bars[st], 1);
    tc::bar_init_fence();
  }

  // B operand: column n = g (heads 0..3 valid), k = dim; the E4 variant uses
  // the permuted dimension order and per-head power-of-two scaling described
  // above score_kernel.
  const bool qok = g < kHI;
  const __nv_bfloat16* qrow = p.qI + (row * kHI + (qok ? g : 0)) * kDI;
  uint32_t bq[4][2];
  int qexp = 0;
  if (E4) {
    const __nv_bfloat16* qp = qrow + t * 16;
    float qv[16];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      qv[i] = qok ? __bfloat162float(qp[i]) : 0.f;
      amax = fmaxf(amax, fabsf(qv[i]));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int e = 14 - (static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127);
    qexp = amax > 0.f ? (e < -60 ? -60 : (e > 60 ? 60 : e)) : 0;
    const float sc = __uint_as_float(static_cast<uint32_t>(qexp + 127) << 23);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      bq[kk][0] = pack_f16x2(qv[4 * kk] * sc, qv[4 * kk + 1] * sc);
      bq[kk][1] = pack_f16x2(qv[4 * kk + 2] * sc, qv[4 * kk + 3] * sc);
    }
  } else {
    const __nv_bfloat16* qp = qrow + t * 2;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      bq[kk][0] = qok ? *reinterpret_cast<const uint32_t*>(qp + kk * 16) : 0u;
      bq[kk][1] = qok ? *reinterpret_cast<const uint32_t*>(qp + kk * 16 + 8) : 0u;
    }
  }
  // accumulator columns 2t, 2t+1 of this lane = heads 2t, 2t+1 (valid for t < 2)
  float w0 = 0.f, w1 = 0.f;
  {
    const int e0 = __shfl_sync(0xffffffffu, qexp, 4 * (2 * t));
    const int e1 = __shfl_sync(0xffffffffu, qexp, 4 * (2 * t + 1));
    if (t < 2) {
      w0 = p.wI[row * kHI + 2 * t] * __uint_as_float(static_cast<uint32_t>(127 - e0) << 23);
      w1 = p.wI[row * kHI + 2 * t + 1] * __uint_as_float(static_cast<uint32_t>(127 - e1) << 23);
    }
  }

  auto load_stage = [&](int tile) {
    const int st = tile % S::kStages;
    const int64_t base = e_begin + static_cast<int64_t>(tile) * kLongTR;
    uint8_t* dst = smem + st * S::kStageBytes;
    if (E4) {
      const int rows = static_cast<int>((e_end - base) < kLongTR ? (e_end - base) : kLongTR);
      if (threadIdx.x == 0) {
        tc::bar_arrive_expect_tx(&bars[st], static_cast<uint32_t>(rows) * 64u);
        tc::bulk_load_stream(dst, p.kcodes + (b * p.N + base) * kDI, static_cast<uint32_t>(rows) * 64u, &bars[st],
                             tc::l2_evict_first_policy());
      }
      const int r = threadIdx.x;  // kLongThreads == kLongTR: one scale per thread
      if (r < rows) {
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(scale_st + st * kLongTR + r)),
                     "l"(p.kscale + b * p.N + base + r));
      } else {
        scale_st[st * kLongTR + r] = 0.f;
      }
      cp_async_commit();
    } else if (threadIdx.x == 0) {
      tc::bar_arrive_expect_tx(&bars[st], static_cast<uint32_t>(S::kStageBytes));
      tc::tma_load_3d_stream(dst, &kmap, 0, static_cast<int>(base), static_cast<int>(b), &bars[st],
                             tc::l2_evict_first_policy());
    }
  };

  __syncthreads();  // barriers initialised, histogram cleared
#pragma unroll
  for (int i = 0; i < S::kStages - 1; ++i) {
    if (i < ntiles) {
      load_stage(i);
    } else if (E4) {
      cp_async_commit();
    }
  }
  // A stage wait that runs out (recorded in the device error word) ends the
  // loop for the whole CTA: no further loads are issued, and the stages still
  // in flight are waited for (again with a bound) before the CTA moves on.
  bool healthy = true;
  int tile = 0;
  for (; tile < ntiles; ++tile) {
    const int st = tile % S::kStages;
    const bool ok = tc::bar_wait(&bars[st], static_cast<uint32_t>((tile / S::kStages) & 1));
    if (E4) cp_async_wait<S::kStages - 2>();
    // every warp is done with the stage refilled next; scales visible
    healthy = __syncthreads_and(ok) != 0;
    if (!healthy) break;
    {
      const int nxt = tile + S::kStages - 1;
      if (nxt < ntiles) {
        load_stage(nxt);
      } else if (E4) {
        cp_async_commit();
      }
    }
    float acc[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
      const int rbase = warp * 32 + mt * 16;
      if (E4) {
        const uint8_t* cs = smem + st * S::kStageBytes + (rbase + g) * 64 + t * 16;
        const uint4 lo = *reinterpret_cast<const uint4*>(cs);
        const uint4 hi = *reinterpret_cast<const uint4*>(cs + 8 * 64);
        const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w}, wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t a0, a1, a2, a3;
          e4m3x4_to_f16x2x2(wl[kk], a0, a2);
          e4m3x4_to_f16x2x2(wh[kk], a1, a3);
          mma_f16(acc[mt], a0, a1, a2, a3, bq[kk][0], bq[kk][1]);
        }
      } else {
        const uint8_t* stg = smem + st * S::kStageBytes;
        const int r = rbase + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int ch = kk * 2 + (lane >> 4);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(a0, a1, a2, a3, stg + r * 128 + ((ch ^ (r & 7)) << 4));
          mma_bf16(acc[mt], a0, a1, a2, a3, bq[kk][0], bq[kk][1]);
        }
      }
    }
    // fold: lanes t = 0, 1 hold heads (0,1) and (2,3) of rows g, g+8 of both
    // tiles; afterwards lane (g, t) owns row 16 (t >> 1) + 8 (t & 1) + g.
    float f[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float part = fmaxf(acc[mt][2 * hf], 0.f) * w0 + fmaxf(acc[mt][2 * hf + 1], 0.f) * w1;
        f[mt][hf] = part + __shfl_xor_sync(0xffffffffu, part, 1);
      }
    }
    const float y = (t & 1) ? f[1][1] : f[1][0];
    const float z = __shfl_xor_sync(0xffffffffu, y, 2);
    float score = t < 2 ? ((t & 1) ? f[0][1] : f[0][0]) : z;
    const int rloc = warp * 32 + (t >> 1) * 16 + (t & 1) * 8 + g;
    if (E4) score *= scale_st[st * kLongTR + rloc];  // scale > 0 factors out of relu
    score += 0.0f;
    const int64_t e = e_begin + static_cast<int64_t>(tile) * kLongTR + rloc;
    if (e < e_end) {
      p.scores[row * p.pitch + e] = score;
      const uint32_t bin = f2key(score) >> 20;
      atomicAdd(&hist_s[bin >> 1], 1u << ((bin & 1u) * 16));
    }
  }
  if (!healthy && threadIdx.x == 0) {
    // stages of tiles [tile, min(ntiles, tile + kStages - 1)) were issued and not consumed
    const int issued_end = (tile + S::kStages - 1) < ntiles ? (tile + S::kStages - 1) : ntiles;
    for (int d = tile; d < issued_end; ++d)
      tc::bar_wait(&bars[d % S::kStages], static_cast<uint32_t>((d / S::kStages) & 1));
  }
  if (E4) cp_async_wait<0>();
  pdl_trigger();  // the next kernel may be scheduled while the histograms merge

  // flush the CTA histogram; the row's last CTA then derives its threshold
  __syncthreads();
  uint32_t* gh = p.hist + row * kHistBins;
  for (int j = threadIdx.x; j < kHistBins / 2; j += kLongThreads) {
    const uint32_t c = hist_s[j];
    if (c & 0xffffu) atomicAdd(gh + 2 * j, c & 0xffffu);
    if (c >> 16) atomicAdd(gh + 2 * j + 1, c >> 16);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t ctas = static_cast<uint32_t>((nv + p.chunk - 1) / p.chunk);
    last_s = (atomicAdd(p.done + 2 * row, 1u) == ctas - 1) ? 1u : 0u;
  }
  __syncthreads();
  if (last_s) {
    __threadfence();
    row_threshold<kLongThreads>(gh, nv, p.k, p.thr + 2 * row, scan_sh);
  }
}

// ---------------------------------------------------------------------------
// row path: one CTA (1024 threads) per query row, row held in shared memory
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) topk_rows_kernel(const float* __restrict__ scores, int64_t N, int64_t Tq,
                                                         int64_t q_pos0, int m, int k, int32_t* __restrict__ idx) {
  pdl_wait();
  pdl_trigger();
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
// The shared-memory bitmap leaves 4 words free after every 16, so that lanes
// reading their 16 consecutive words as four 16-byte vectors (the emission
// pass) do not collide on banks.
__host__ __device__ constexpr int bm_pad(int64_t wi) { return static_cast<int>(wi + 4 * (wi >> 4)); }
constexpr int kBitmapSmemPadded = kBitmapSmemWords + kBitmapSmemWords / 4;

struct LongWs {
  float* scores;        // [R, pitch] (pitch = N rounded up to 4: 16-byte aligned rows)
  uint32_t* hist;       // [R, kHistBins]    (zeroed per call)
  uint32_t* cand_cnt;   // [R]               (zeroed per call)
  uint32_t* done;       // [R, 2]: scoring / select CTAs finished (zeroed per call)
  int32_t* thr;         // [R, 2]
  uint2* cand;          // [R, N]: (key, index) of the threshold bin's entries
  uint32_t* bitmap;     // [R, W]
  int64_t W;
  int64_t pitch;
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
  pdl_wait();
  extern __shared__ __align__(16) uint8_t sel_smem[];  // candidates, then the final bitmap
  uint2* cand_s = reinterpret_cast<uint2*>(sel_smem);
  uint32_t* bm_s = reinterpret_cast<uint32_t*>(sel_smem + kCandSmem * sizeof(uint2));
  __shared__ uint32_t hist[256];
  __shared__ uint32_t dig[3];
  __shared__ uint32_t n_cand, base_s, last_s;
  const int64_t row = blockIdx.y;
  const int64_t nv = visible(q_pos0 + row % Tq, m, N);
  const int64_t e_begin = static_cast<int64_t>(blockIdx.x) * kSelChunk;
  int32_t* out = idx + row * k;
  if (nv == 0) {  // no entry visible yet (the scoring kernel skipped the row): all padding
    if (blockIdx.x == 0) write_prefix_ids(out, 0, k);
    return;
  }
  if (e_begin >= nv) return;
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
  // warp w scans entries [e_begin + 512 w, e_begin + 512 (w + 1)), four per
  // lane per step (16-byte loads; rows are 16-byte aligned and padded)
  const float* srow = ws.scores + row * ws.pitch;
  constexpr int kSelWarps = kSelThreads / 32;
  constexpr int kPerWarp = kSelChunk / kSelWarps;
  constexpr int kSteps = kPerWarp / 128;
  const int warp = threadIdx.x >> 5;
  float4 sv[kSteps];
#pragma unroll
  for (int it = 0; it < kSteps; ++it) {  // all loads first, then the bookkeeping
    const int64_t i = e_begin + warp * kPerWarp + it * 128 + 4 * lane;
    sv[it] = i < e_end ? __ldcg(reinterpret_cast<const float4*>(srow + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int it = 0; it < kSteps; ++it) {
    const int64_t base = e_begin + warp * kPerWarp + it * 128;  // a multiple of 32
    if (base >= e_end) break;                                     // uniform for the warp
    const int64_t i0 = base + 4 * lane;
    const float v[4] = {sv[it].x, sv[it].y, sv[it].z, sv[it].w};
    uint32_t above = 0, cand_bits = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const bool ok = i0 + u < e_end;
      const uint32_t bin = f2key(v[u]) >> 20;
      above |= (ok && bin > tb) ? (1u << u) : 0u;
      cand_bits |= (ok && bin == tb) ? (1u << u) : 0u;
    }
    // bitmap word of entries [32 j, 32 j + 32): lanes 8j .. 8j+7, four bits each
    uint32_t word = above << (4 * (lane & 7));
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    word |= __shfl_xor_sync(0xffffffffu, word, 4);
    if ((lane & 7) == 0 && i0 < e_end) ws.bitmap[row * ws.W + (i0 >> 5)] = word;
    if (__any_sync(0xffffffffu, cand_bits != 0u)) {
      const uint32_t nc = __popc(cand_bits);
      uint32_t incl = nc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      uint32_t pos = 0;
      if (lane == 31) pos = atomicAdd(&n_cand, incl);
      pos = __shfl_sync(0xffffffffu, pos, 31) + incl - nc;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (cand_bits & (1u << u)) {
          const uint2 kv = make_uint2(f2key(v[u]), static_cast<uint32_t>(i0 + u));
          if (pos < static_cast<uint32_t>(kCandSmem)) {
            cand_s[pos] = kv;
          } else {  // rare (many equal scores): straight to the row's list
            ws.cand[row * N + atomicAdd(ws.cand_cnt + row, 1u)] = kv;
          }
          ++pos;
        }
      }
    }
  }
  __syncthreads();
  const uint32_t nc = n_cand < static_cast<uint32_t>(kCandSmem) ? n_cand : static_cast<uint32_t>(kCandSmem);
  if (threadIdx.x == 0 && nc) base_s = atomicAdd(ws.cand_cnt + row, nc);
  __syncthreads();
  for (uint32_t c = threadIdx.x; c < nc; c += kSelThreads) ws.cand[row * N + base_s + c] = cand_s[c];
  pdl_trigger();  // only the rows' last CTAs still have work
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

  // ---- load the row's candidates (when they fit) and bitmap (when it fits)
  // together.  Warp w owns the bitmap words [w * per_warp, (w + 1) * per_warp)
  // and counts their bits as it loads them (wcnt), so the final emission
  // needs no separate counting pass.
  const int64_t words = (nv + 31) >> 5;
  const uint32_t cnt = __ldcg(ws.cand_cnt + row);
  const uint2* cand = ws.cand + row * N;
  uint32_t* gbm = ws.bitmap + row * ws.W;
  const bool bm_in_smem = words <= kBitmapSmemWords;
  const bool cand_in_smem = cnt <= static_cast<uint32_t>(kCandSmem);
  __shared__ uint32_t wcnt[kSelWarps];
  // a shared-memory bitmap gives every warp 512 words (16 per lane)
  const int64_t per_warp =
      bm_in_smem ? kBitmapSmemWords / kSelWarps : (words + 32 * kSelWarps - 1) / (32 * kSelWarps) * 32;
  const int64_t wb = warp * per_warp;
  const int64_t we = (wb + per_warp) < words ? (wb + per_warp) : words;
  // candidate loads first (in flight together with the bitmap's)
  constexpr int kCandPerThread = kCandSmem / kSelThreads;
  uint2 cv[kCandPerThread];
  if (cand_in_smem) {
#pragma unroll
    for (int u = 0; u < kCandPerThread; ++u) {
      const uint32_t c = u * kSelThreads + threadIdx.x;
      cv[u] = c < cnt ? __ldcg(cand + c) : make_uint2(0, 0);
    }
  }
  {
    // 16 words per lane in flight (a shared-memory bitmap has at most 512 words per warp)
    uint32_t bits = 0;
    for (int64_t w0 = wb; w0 < we; w0 += 16 * 32) {
      uint32_t v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int64_t wi = w0 + u * 32 + lane;
        v[u] = wi < we ? __ldcg(gbm + wi) : 0u;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int64_t wi = w0 + u * 32 + lane;
        if (wi == words - 1 && (nv & 31)) v[u] &= (1u << (nv & 31)) - 1u;
        if (bm_in_smem && wi < we) bm_s[bm_pad(wi)] = v[u];
        bits += __popc(v[u]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bits += __shfl_xor_sync(0xffffffffu, bits, o);
    if (lane == 0) wcnt[warp] = bits;
  }
  if (cand_in_smem) {
#pragma unroll
    for (int u = 0; u < kCandPerThread; ++u) {
      const uint32_t c = u * kSelThreads + threadIdx.x;
      if (c < cnt) cand_s[c] = cv[u];
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
  for (uint32_t c = threadIdx.x; c < cnt; c += kSelThreads) {
    const uint2 kv = cand_in_smem ? cand[c] : __ldcg(cand + c);
    const uint64_t x = (static_cast<uint64_t>(kv.x) << 32) | (0xffffffffu - kv.y);
    if ((x & mask) >= prefix) {  // a threshold-bin entry: its bit is not set yet
      atomicOr(bm_in_smem ? bm_s + bm_pad(kv.y >> 5) : gbm + (kv.y >> 5), 1u << (kv.y & 31));
      atomicAdd(&wcnt[(kv.y >> 5) / per_warp], 1u);
    }
  }
  if (!bm_in_smem) __threadfence();
  __syncthreads();

  // ---- ascending list from the bitmap: each warp emits its own word range
  // at the offset of the bits before it; within the warp each lane takes
  // per_warp / 32 consecutive words (one count pass, one scan, one emit pass).
  uint32_t pos = 0;
  for (int w = 0; w < warp; ++w) pos += wcnt[w];
  const int64_t per_lane = per_warp / 32;
  const int64_t lb = wb + lane * per_lane;
  const int64_t le = (lb + per_lane) < we ? (lb + per_lane) : we;
  if (bm_in_smem) {  // 16 words per lane, in registers
    static_assert(kBitmapSmemWords / kSelWarps == 16 * 32, "16 bitmap words per lane");
    uint32_t wv[16];
    const uint4* src = reinterpret_cast<const uint4*>(bm_s + bm_pad(lb));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 v = src[j];
      wv[4 * j] = v.x;
      wv[4 * j + 1] = v.y;
      wv[4 * j + 2] = v.z;
      wv[4 * j + 3] = v.w;
    }
    uint32_t c = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int64_t wi = lb + j;
      if (wi >= words) wv[j] = 0u;
      if (wi == words - 1 && (nv & 31)) wv[j] &= (1u << (nv & 31)) - 1u;
      c += __popc(wv[j]);
    }
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    uint32_t p = pos + incl - c;
    const int32_t e0 = static_cast<int32_t>(lb << 5);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      uint32_t word = wv[j];
      while (word) {
        const int bit = __ffs(word) - 1;
        word &= word - 1;
        if (p < static_cast<uint32_t>(k)) out[p] = e0 + 32 * j + bit;
        ++p;
      }
    }
    return;
  }
  uint32_t c = 0;
  for (int64_t wi = lb; wi < le; ++wi) {
    uint32_t word = __ldcg(gbm + wi);
    if (wi == words - 1 && (nv & 31)) word &= (1u << (nv & 31)) - 1u;
    c += __popc(word);
  }
  uint32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  uint32_t p = pos + incl - c;
  for (int64_t wi = lb; wi < le && p < static_cast<uint32_t>(k); ++wi) {
    uint32_t word = __ldcg(gbm + wi);
    if (wi == words - 1 && (nv & 31)) word &= (1u << (nv & 31)) - 1u;
    while (word) {
      const int bit = __ffs(word) - 1;
      word &= word - 1;
      if (p < static_cast<uint32_t>(k)) out[p] = static_cast<int32_t>((wi << 5) + bit);
      ++p;
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool use_row_path(int64_t R, int64_t N) { return N <= kRowPathMaxN && R > 256; }

struct LongLayout {
  size_t scores, hist, cnt, done, thr, cand, bitmap, total;
  int64_t W, pitch;
};

LongLayout long_layout(int64_t R, int64_t N) {
  LongLayout L;
  L.W = ((N + 31) / 32 + 15) / 16 * 16;  // 16-word multiple: vector reads stay in the row
  L.pitch = (N + 3) / 4 * 4;
  size_t off = 0;
  L.scores = off; off = align_up(off + static_cast<size_t>(R) * L.pitch * 4);
  L.hist = off;   off += static_cast<size_t>(R) * kHistBins * 4;     // hist, cnt and done: zeroed together
  L.cnt = off;    off += static_cast<size_t>(R) * 4;
  L.done = off;   off = align_up(off + static_cast<size_t>(R) * 8);
  L.thr = off;    off = align_up(off + static_cast<size_t>(R) * 8);
  L.cand = off;   off = align_up(off + static_cast<size_t>(R) * N * 8);
  L.bitmap = off; off = align_up(off + static_cast<size_t>(R) * L.W * 4);
  L.total = off;
  return L;
}

// Query rows B * Tq, or -1 when B or Tq is negative or the product is not
// below 2^31 (checked before multiplying, so it cannot overflow).
int64_t query_rows(int64_t B, int64_t Tq) {
  constexpr int64_t kLim = int64_t(1) << 31;
  if (B < 0 || Tq < 0 || B >= kLim || Tq >= kLim) return -1;
  if (Tq > 0 && B > (kLim - 1) / Tq) return -1;
  return B * Tq;
}

size_t workspace_bytes(int64_t B, int64_t Tq, int64_t N) {
  const int64_t R = query_rows(B, Tq);
  if (R <= 0 || N <= 0 || N >= (int64_t(1) << 31)) return 0;
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

}  // extern "C"

namespace csa {
namespace {
csa_status indexer_impl(const void* qI, const float* wI, const void* kIc, const uint8_t* kcodes, const float* kscale,
                        int64_t B, int64_t Tq, int64_t N, int64_t q_pos0, int32_t m, int32_t k, int32_t* idx,
                        void* workspace, size_t workspace_bytes, void* stream) {
  clear_error();
  const bool e4 = kcodes != nullptr;
  CSA_REQUIRE(B >= 0 && Tq >= 0 && N >= 0, "csa_indexer_topk: negative size");
  CSA_REQUIRE(N < (1LL << 31), "csa_indexer_topk: N must be < 2^31");
  CSA_REQUIRE(m >= 1, "csa_indexer_topk: m must be >= 1");
  CSA_REQUIRE(k >= 1 && k <= kMaxK, "csa_indexer_topk: k must be in [1, %d] (got %d)", kMaxK, k);
  CSA_REQUIRE(q_pos0 >= 0 && q_pos0 < (int64_t(1) << 50), "csa_indexer_topk: q_pos0 must be in [0, 2^50)");
  const int64_t R = query_rows(B, Tq);
  CSA_REQUIRE(R >= 0, "csa_indexer_topk: B * Tq must be below 2^31");
  if (R == 0) return CSA_OK;
  CSA_REQUIRE_PTR(idx);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (N == 0) {
    if (cudaMemsetAsync(idx, 0xff, static_cast<size_t>(R) * k * 4, s) != cudaSuccess)
      return fail(CSA_ERR_CUDA, "csa_indexer_topk: memset failed");
    return CSA_OK;
  }
  CSA_REQUIRE_PTR(qI);
  CSA_REQUIRE_PTR(wI);
  if (e4) {
    CSA_REQUIRE_PTR(kcodes);
    CSA_REQUIRE(kscale != nullptr && (reinterpret_cast<uintptr_t>(kscale) & 3u) == 0,
                "csa_indexer_topk: key scales NULL or misaligned");
  } else {
    CSA_REQUIRE_PTR(kIc);
  }
  const size_t need = csa::workspace_bytes(B, Tq, N);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "csa_indexer_topk: workspace of %zu bytes needed (got %zu)", need,
                workspace_bytes);
  CSA_REQUIRE(aligned16(workspace), "csa_indexer_topk: workspace is not 16-byte aligned");

  ScoreParams p;
  p.qI = static_cast<const __nv_bfloat16*>(qI);
  p.wI = wI;
  p.kI = static_cast<const __nv_bfloat16*>(kIc);
  p.kcodes = kcodes;
  p.kscale = kscale;
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
    const cudaError_t e = e4 ? launch_pdl(score_kernel<QR, true>, grid, dim3(kScoreThreads), score_tile_bytes(true), s, 1, p)
                             : launch_pdl(score_kernel<QR, false>, grid, dim3(kScoreThreads), tile_smem, s, 1, p);
    prof_end(s);
    if (csa_status st = check_launch("indexer score", e); st != CSA_OK) return st;
    const size_t smem = static_cast<size_t>(N) * 4;
    if (!ensure_smem(reinterpret_cast<const void*>(topk_rows_kernel), kRowPathMaxN * 4))
      return fail(CSA_ERR_CUDA, "csa_indexer_topk: cannot raise shared memory limit");
    return check_launch("indexer top-k (rows)",
                        launch_pdl(topk_rows_kernel, dim3(static_cast<unsigned>(R)), dim3(1024), smem, s, 1,
                                   static_cast<const float*>(p.scores), N, Tq, q_pos0, m, k, idx));
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
  w.pitch = L.pitch;
  if (cudaMemsetAsync(w.hist, 0, L.thr - L.hist, s) != cudaSuccess)
    return fail(CSA_ERR_CUDA, "csa_indexer_topk: memset failed");
  CSA_REQUIRE(R < 65536, "csa_indexer_topk: too many query rows for the long-row path");
  LongScoreParams lp;
  lp.qI = p.qI;
  lp.wI = wI;
  lp.kcodes = kcodes;
  lp.kscale = kscale;
  lp.Tq = Tq;
  lp.N = N;
  lp.q_pos0 = q_pos0;
  lp.m = m;
  lp.scores = w.scores;
  lp.pitch = w.pitch;
  lp.hist = w.hist;
  lp.done = w.done;
  lp.thr = w.thr;
  lp.k = k;
  CUtensorMap kmap;
  memset(&kmap, 0, sizeof(kmap));
  if (!e4) {
    const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (encode == nullptr) return fail(CSA_ERR_CUDA, "csa_indexer_topk: cuTensorMapEncodeTiled unavailable");
    CSA_REQUIRE(aligned16(kIc), "csa_indexer_topk: kIc must be 16-byte aligned");
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDI), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDI) * 2, static_cast<cuuint64_t>(N) * kDI * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kDI), static_cast<cuuint32_t>(kLongTR), 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUresult r = encode(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kIc), dims,
                                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CSA_ERR_CUDA, "csa_indexer_topk: tensor map encoding failed (%d)", int(r));
  } else {
    CSA_REQUIRE(aligned16(kcodes), "csa_indexer_topk: key codes must be 16-byte aligned");
  }
  const void* skern = e4 ? reinterpret_cast<const void*>(score_long_kernel<true>)
                        : reinterpret_cast<const void*>(score_long_kernel<false>);
  const size_t ssmem = e4 ? LongShape<true>::kSmem : LongShape<false>::kSmem;
  if (!ensure_smem(skern, static_cast<int>(ssmem)))
    return fail(CSA_ERR_CUDA, "csa_indexer_topk: cannot raise shared memory limit");
  // one wave: the row's chunks spread over every resident CTA slot
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, skern, kLongThreads, ssmem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t per_row = std::max<int64_t>(1, static_cast<int64_t>(num_sms()) * per_sm / R);
  int64_t chunk = (N + per_row - 1) / per_row;
  chunk = std::max<int64_t>(kLongMinChunk, (chunk + kLongTR - 1) / kLongTR * kLongTR);
  chunk = std::min<int64_t>(chunk, kLongMaxChunk);
  lp.chunk = static_cast<int>(chunk);
  dim3 grid(static_cast<unsigned>((N + chunk - 1) / chunk), static_cast<unsigned>(R));
  prof_begin(s);
  const cudaError_t e = e4 ? launch_pdl(score_long_kernel<true>, grid, dim3(kLongThreads), ssmem, s, 1, lp, kmap)
                           : launch_pdl(score_long_kernel<false>, grid, dim3(kLongThreads), ssmem, s, 1, lp, kmap);
  prof_end(s);
  if (csa_status st = check_launch("indexer score (long rows)", e); st != CSA_OK) return st;
  dim3 sgrid(static_cast<unsigned>((N + kSelChunk - 1) / kSelChunk), static_cast<unsigned>(R));
  constexpr int kSelSmem = kCandSmem * 8 + kBitmapSmemPadded * 4;
  if (!ensure_smem(reinterpret_cast<const void*>(topk_select_kernel), kSelSmem))
    return fail(CSA_ERR_CUDA, "csa_indexer_topk: cannot raise shared memory limit");
  return check_launch("indexer select",
                      launch_pdl(topk_select_kernel, sgrid, dim3(kSelThreads), kSelSmem, s, 1, w, N, Tq, q_pos0, m, k, idx));
}
}  // namespace
}  // namespace csa

extern "C" {

csa_status csa_indexer_topk(const void* qI, const float* wI, const void* kIc, int64_t B, int64_t Tq, int64_t N,
                            int64_t q_pos0, int32_t m, int32_t k, int32_t* idx, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return csa::indexer_impl(qI, wI, kIc, nullptr, nullptr, B, Tq, N, q_pos0, m, k, idx, workspace, workspace_bytes,
                           stream);
}

csa_status csa_indexer_topk_e4m3(const void* qI, const float* wI, const uint8_t* kI_codes, const float* kI_scale,
                                 int64_t B, int64_t Tq, int64_t N, int64_t q_pos0, int32_t m, int32_t k, int32_t* idx,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  return csa::indexer_impl(qI, wI, nullptr, kI_codes, kI_scale, B, Tq, N, q_pos0, m, k, idx, workspace,
                           workspace_bytes, stream);
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
// (on the host it is only a stand-in for the symbol), so every call looks up
// the array's device address with cudaGetSymbolAddress on the current device;
// the first call on a device may also load the library's device code there,
// so make that first call before any stream capture.  The call itself
// allocates nothing: it forwards
// to csa_indexer_topk with the cached address as the workspace, and that path
// clears the parts of the scratch that must start at zero on every call.  All
// calls share the one array and it keeps the last call's contents, so calls
// that overlap on the GPU (different streams, or host threads, without
// ordering between them) race on it.
// ---------------------------------------------------------------------------
static constexpr size_t kStaticScratchBytes = static_cast<size_t>(32) << 20;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

extern "C" csa_status csa_indexer_topk_noalloc(const void* qI, const float* wI, const void* kIc, int64_t B,
                                               int64_t Tq, int64_t N, int64_t q_pos0, int32_t m, int32_t k,
                                               int32_t* idx, void* stream) {
  using namespace csa;
  if (B < 0 || Tq < 0 || N < 0) return fail(CSA_ERR_INVALID_ARG, "csa_indexer_topk_noalloc: negative size");
  if (query_rows(B, Tq) < 0 || N >= (int64_t(1) << 31))
    return fail(CSA_ERR_INVALID_ARG, "csa_indexer_topk_noalloc: B * Tq and N must be below 2^31");
  const size_t need = csa::workspace_bytes(B, Tq, N);
  if (need > kStaticScratchBytes)
    return fail(CSA_ERR_UNSUPPORTED,
                "csa_indexer_topk_noalloc: these sizes need %zu bytes of scratch but the static scratch holds %zu; "
                "call csa_indexer_topk with a caller workspace instead",
                need, kStaticScratchBytes);
  void* ptr = nullptr;
  if (need > 0) {
    // looked up on every call (a host-side query that allocates nothing), so a
    // device reset or a new primary context never leaves a stale address behind
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess)
      return fail(CSA_ERR_CUDA, "csa_indexer_topk_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
  }
  return csa_indexer_topk(qI, wI, kIc, B, Tq, N, q_pos0, m, k, idx, ptr, ptr ? kStaticScratchBytes : 0, stream);
}
