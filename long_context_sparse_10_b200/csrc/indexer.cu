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
//     the key's top 12 bits fused into the scoring kernel; a classifying
//     kernel then derives each row's threshold bin from it (in every CTA) and
//     emits a bitmap of the entries above that bin, their count per chunk and
//     a candidate list of the bin itself; an emitting kernel resolves the cut
//     among the candidates (in every CTA of the row) and writes the ascending
//     list, each CTA its own span of the row.  No CTA ever waits for another.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "host_util.h"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int kMaxK = 4096;
// Key formats of the scoring kernels: bf16 keys, or coded keys with one fp32
// scale per entry -- E4M3 (64 bytes per entry) or E2M1 (FP4, 32 bytes).
constexpr int kKeyBF16 = 0, kKeyE4M3 = 1, kKeyE2M1 = 2;
__host__ __device__ constexpr int code_bytes(int kf) { return kf == kKeyE2M1 ? 32 : 64; }
constexpr int kRowPathMaxN = 32768;  // rows up to this many visible entries live in shared memory
constexpr int kHistBins = 4096;      // first-level bins: top 12 bits of the key
constexpr int kErrRowTooLong = 2;    // device error word: a row-path row longer than its shared memory
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
  int64_t pitch;    // row pitch of scores (N, or the longest packed sequence's entries)
  // packed sequences (nullable): sequence s owns query rows [cu_tok[s],
  // cu_tok[s+1]) (positions from 0) and key rows [cu_ent[s], cu_ent[s+1]);
  // CTA row y of the grid is the s-th sequence's group y - cu_grp[s] of QR rows
  const int32_t* cu_tok;
  const int32_t* cu_ent;
  const int32_t* cu_grp;
  int n_seqs;
};

__device__ __forceinline__ void named_sync_ix(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

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

// The whole visible prefix [0, nv) selected (nv <= k), -1 padded; with a
// score output, each slot also gets the entry's score (-inf for padding).
__device__ __forceinline__ void write_prefix_ids(int32_t* out, int64_t nv, int k, float* sout = nullptr,
                                                 const float* srow = nullptr) {
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    out[j] = j < nv ? j : -1;
    if (sout != nullptr) sout[j] = j < nv ? __ldcg(srow + j) : -INFINITY;
  }
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
__host__ __device__ constexpr size_t score_tile_bytes(int kf) {
  return kf != kKeyBF16 ? static_cast<size_t>(kStages) * (2 * kTileRows) * (code_bytes(kf) + 4)
                        : static_cast<size_t>(kStages) * kTileRows * 128;
}

// A fragments (fp16) of one 16-entry MMA tile of coded keys for k-step kk:
// the lane's entry row g (codes at `row`) and g + 8, dimensions 16t + 4kk ..
// 16t + 4kk + 3 (the permuted order described below).
template <int KF>
__device__ __forceinline__ void key_frags(const uint8_t* row, int t, uint32_t (&af)[4][4]) {
  constexpr int CB = code_bytes(KF);
  if constexpr (KF == kKeyE4M3) {  // 16 codes = dims 16t .. 16t+15, one byte each
    const uint4 lo = *reinterpret_cast<const uint4*>(row + t * 16);
    const uint4 hi = *reinterpret_cast<const uint4*>(row + 8 * CB + t * 16);
    const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w}, wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      e4m3x4_to_f16x2x2(wl[kk], af[kk][0], af[kk][2]);
      e4m3x4_to_f16x2x2(wh[kk], af[kk][1], af[kk][3]);
    }
  } else {  // E2M1: 8 bytes = dims 16t .. 16t+15, two per byte (low nibble = even dim)
    const uint2 lo = *reinterpret_cast<const uint2*>(row + t * 8);
    const uint2 hi = *reinterpret_cast<const uint2*>(row + 8 * CB + t * 8);
    const uint32_t wl[2] = {lo.x, lo.y}, wh[2] = {hi.x, hi.y};
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint16_t bl = static_cast<uint16_t>(wl[kk >> 1] >> (16 * (kk & 1)));
      const uint16_t bh = static_cast<uint16_t>(wh[kk >> 1] >> (16 * (kk & 1)));
      e2m1x4_to_f16x2x2(bl, af[kk][0], af[kk][2]);
      e2m1x4_to_f16x2x2(bh, af[kk][1], af[kk][3]);
    }
  }
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
template <int QR, int KF>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(ScoreParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr bool E4 = KF != kKeyBF16;  // coded keys (E4M3 or E2M1) with a per-entry scale
  constexpr int CB = code_bytes(KF);   // code bytes per entry
  constexpr int NCOL = QR * 4;
  constexpr int NT = (NCOL + 7) / 8;
  constexpr int TR = E4 ? 2 * kTileRows : kTileRows;  // entries per stage
  constexpr int MT = TR / kTileRows;                  // 16-row MMA tiles per warp and stage
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* tiles = smem;                                             // bf16: [kStages] swizzled tiles
  uint8_t* codes_st = smem;                                          // coded: [kStages][TR][CB]
  float* scale_st = reinterpret_cast<float*>(smem + kStages * TR * CB);  // coded: [kStages][TR]

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // this CTA's QR query rows: global rows qrow0.., positions t0.., keys ebase.. (Nseq of them)
  int64_t qrow0, t0, ebase, Nseq;
  int nrows;
  if (p.cu_tok != nullptr) {
    const int64_t gy = blockIdx.y;
    if (gy >= __ldg(p.cu_grp + p.n_seqs)) return;
    const int sq = seq_of(p.cu_grp, p.n_seqs, gy);
    const int64_t len = __ldg(p.cu_tok + sq + 1) - __ldg(p.cu_tok + sq);
    t0 = (gy - __ldg(p.cu_grp + sq)) * QR;
    qrow0 = __ldg(p.cu_tok + sq) + t0;
    nrows = static_cast<int>((len - t0) < QR ? (len - t0) : QR);
    ebase = __ldg(p.cu_ent + sq);
    Nseq = __ldg(p.cu_ent + sq + 1) - ebase;
  } else {
    const int64_t groups = (p.Tq + QR - 1) / QR;
    const int64_t b = blockIdx.y / groups;
    const int64_t r0 = (blockIdx.y % groups) * QR;
    qrow0 = b * p.Tq + r0;
    t0 = p.q_pos0 + r0;
    nrows = static_cast<int>((p.Tq - r0) < QR ? (p.Tq - r0) : QR);
    ebase = b * p.N;
    Nseq = p.N;
  }
  const int64_t nv_max = visible(t0 + nrows - 1, p.m, Nseq);
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
    const __nv_bfloat16* qrow = p.qI + (((qrow0 + (ok ? rr : 0)) * kHI + h) * kDI);
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
    const int64_t row = qrow0 + (ok ? rr : 0);
    const int h0 = (lane & 1) * 2;
    wv[nt][0] = ok ? p.wI[row * kHI + h0] : 0.f;
    wv[nt][1] = ok ? p.wI[row * kHI + h0 + 1] : 0.f;
    if (E4) {  // columns 2t, 2t+1 of this n-tile were scaled by the lanes with g = 2t, 2t+1
      const int e0 = __shfl_sync(0xffffffffu, qexp[nt], 4 * (2 * (lane & 3)));
      const int e1 = __shfl_sync(0xffffffffu, qexp[nt], 4 * (2 * (lane & 3) + 1));
      wv[nt][0] *= __uint_as_float(static_cast<uint32_t>(127 - e0) << 23);
      wv[nt][1] *= __uint_as_float(static_cast<uint32_t>(127 - e1) << 23);
    }
    nv_r[nt] = ok ? visible(t0 + rr, p.m, Nseq) : 0;
    srow[nt] = row;
  }

  const int ntiles = static_cast<int>((e_end - e_begin + TR - 1) / TR);
  const __nv_bfloat16* kbase = p.kI + ebase * kDI;
  auto load_tile = [&](int tile, int stage) {
    const int64_t base = e_begin + static_cast<int64_t>(tile) * TR;
    if constexpr (E4) {
      // CB code bytes per entry (CB / 16 pieces) and one 4-byte scale per entry
      constexpr int PPE = CB / 16;
      for (int piece = threadIdx.x; piece < TR * PPE; piece += kScoreThreads) {
        const int row = piece / PPE, ch = piece % PPE;
        const int64_t e = base + row;
        const bool ok = e < e_end;
        cp_async16(codes_st + (stage * TR + row) * CB + ch * 16,
                   p.kcodes + (ebase + (ok ? e : e_begin)) * CB + ch * 16, ok ? 16 : 0);
      }
      for (int row = threadIdx.x; row < TR; row += kScoreThreads) {
        const int64_t e = base + row;
        if (e < e_end) {
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(scale_st + stage * TR + row)),
                       "l"(p.kscale + ebase + e));
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
        uint32_t af[4][4];
        key_frags<KF>(codes_st + ((tile % kStages) * TR + rbase + (lane >> 2)) * CB, lane & 3, af);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_f16(acc[nt], af[kk][0], af[kk][1], af[kk][2], af[kk][3], bq[kk][nt][0], bq[kk][nt][1]);
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
            p.scores[srow[nt] * p.pitch + e] = full;
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
template <int KF>
struct LongShape {
  static constexpr bool E4 = KF != kKeyBF16;
  static constexpr int kStages = E4 ? CSA_LONG_STAGES_E4 : CSA_LONG_STAGES_BF16;
  static constexpr int kStageBytes = kLongTR * (E4 ? code_bytes(KF) : 128);
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
  uint32_t* hist;  // [R, kHistBins] (zeroed per call): each CTA adds its chunk's bins
  int k;
};

template <int KF>
__global__ void __launch_bounds__(kLongThreads) score_long_kernel(LongScoreParams p,
                                                                  const __grid_constant__ CUtensorMap kmap) {
  pdl_wait();
  using S = LongShape<KF>;
  constexpr bool E4 = S::E4;  // coded keys (E4M3 or E2M1) with a per-entry scale
  constexpr int CB = code_bytes(KF);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float* scale_st = reinterpret_cast<float*>(smem + S::kScaleOff);  // E4: [kStages][kLongTR]
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + S::kHistOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBarOff);

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
        tc::bar_arrive_expect_tx(&bars[st], static_cast<uint32_t>(rows) * CB);
        tc::bulk_load_stream(dst, p.kcodes + (b * p.N + base) * CB, static_cast<uint32_t>(rows) * CB, &bars[st],
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
        uint32_t af[4][4];
        key_frags<KF>(smem + st * S::kStageBytes + (rbase + g) * CB, t, af);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_f16(acc[mt], af[kk][0], af[kk][1], af[kk][2], af[kk][3], bq[kk][0], bq[kk][1]);
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

  // flush the CTA histogram
  __syncthreads();
  uint32_t* gh = p.hist + row * kHistBins;
  for (int j = threadIdx.x; j < kHistBins / 2; j += kLongThreads) {
    const uint32_t c = hist_s[j];
    if (c & 0xffffu) atomicAdd(gh + 2 * j, c & 0xffffu);
    if (c >> 16) atomicAdd(gh + 2 * j + 1, c >> 16);
  }
  // (the classifying kernel derives each row's threshold from the complete
  // histogram once this grid has finished: no counter, no waiting CTA)
}

// ---------------------------------------------------------------------------
// row path: one CTA (1024 threads) per query row, row held in shared memory
// ---------------------------------------------------------------------------
struct RowsParams {
  const float* scores;
  int64_t pitch, N, Tq, q_pos0;
  int m, k;
  int32_t* idx;
  const int32_t* cu_tok;  // packed sequences (nullable): as ScoreParams
  const int32_t* cu_ent;
  int n_seqs;
  float* sout;            // nullable: [R, k] score of each selected entry
};

__global__ void __launch_bounds__(1024) topk_rows_kernel(RowsParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t dig[3];
  __shared__ uint32_t scan_sh[32];
  const int64_t row = blockIdx.x;
  int64_t nv;
  if (p.cu_tok != nullptr) {
    const int sq = seq_of(p.cu_tok, p.n_seqs, row);
    nv = visible(row - __ldg(p.cu_tok + sq), p.m, __ldg(p.cu_ent + sq + 1) - __ldg(p.cu_ent + sq));
  } else {
    nv = visible(p.q_pos0 + row % p.Tq, p.m, p.N);
  }
  const int k = p.k;
  int32_t* out = p.idx + row * k;
  float* sout = p.sout != nullptr ? p.sout + row * k : nullptr;
  const float* srow = p.scores + row * p.pitch;
  if (nv <= k) {
    write_prefix_ids(out, nv, k, sout, srow);
    return;
  }
  if (nv > kRowPathMaxN) {  // cannot happen for sizes the host admits; never index past the shared row
    if (threadIdx.x == 0) atomicExch(&tc::g_device_error, kErrRowTooLong);
    write_prefix_ids(out, 0, k, sout, srow);
    return;
  }
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
    if (sel) {
      out[pos] = static_cast<int32_t>(i);
      if (sout != nullptr) sout[pos] = srow[i];
    }
    ties_before += tie_total;
    sel_before += sel_total;
  }
}

// Short rows (at most 1024 visible entries): one warp per row, 32 consecutive
// entries per lane in registers; the same exact radix select (four levels of
// 8 key bits, a 256-bin histogram per warp in shared memory, the threshold
// digit found by a warp scan over the bins from the top), then an ascending
// emission: lane order is index order, so warp scans of the per-lane counts
// give every selected entry its position and the ties their rank.
constexpr int kWarpRowMaxN = 1024;

__global__ void __launch_bounds__(256) topk_rows_warp_kernel(RowsParams p, int64_t R) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t hist_all[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  if (row >= R) return;  // whole warps only: nothing below synchronises the block
  uint32_t* hist = hist_all[warp];
  int64_t nv;
  if (p.cu_tok != nullptr) {
    const int sq = seq_of(p.cu_tok, p.n_seqs, row);
    nv = visible(row - __ldg(p.cu_tok + sq), p.m, __ldg(p.cu_ent + sq + 1) - __ldg(p.cu_ent + sq));
  } else {
    nv = visible(p.q_pos0 + row % p.Tq, p.m, p.N);
  }
  const int k = p.k;
  int32_t* out = p.idx + row * k;
  float* sout = p.sout != nullptr ? p.sout + row * k : nullptr;
  const float* srow = p.scores + row * p.pitch;
  if (nv <= k || nv > kWarpRowMaxN) {
    if (nv > k && lane == 0) atomicExch(&tc::g_device_error, kErrRowTooLong);  // the host never admits this
    const int64_t keep = nv <= k ? nv : 0;
    for (int j = lane; j < k; j += 32) {
      out[j] = j < keep ? j : -1;
      if (sout != nullptr) sout[j] = j < keep ? __ldcg(srow + j) : -INFINITY;
    }
    return;
  }
  const int n = static_cast<int>(nv), base = lane * 32;
  uint32_t key[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) key[i] = base + i < n ? f2key(__ldcg(srow + base + i)) : 0u;
  uint32_t prefix = 0, mask = 0, remaining = static_cast<uint32_t>(k);
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int j = lane; j < 256; j += 32) hist[j] = 0u;
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (base + i < n && (key[i] & mask) == prefix) atomicAdd(&hist[(key[i] >> shift) & 255u], 1u);
    __syncwarp();
    // lane l owns bins 255 - 8l .. 248 - 8l (descending)
    uint32_t c[8], tot = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      c[j] = hist[255 - 8 * lane - j];
      tot += c[j];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t excl = incl - tot;
    const int owner = __ffs(__ballot_sync(0xffffffffu, excl < remaining && remaining <= incl)) - 1;
    uint32_t digit = 0, above = 0;
    if (lane == owner) {
      uint32_t run = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (run + c[j] >= remaining) {
          digit = static_cast<uint32_t>(255 - 8 * lane - j);
          above = run;
          break;
        }
        run += c[j];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, owner);
    above = __shfl_sync(0xffffffffu, above, owner);
    prefix |= digit << shift;
    mask |= 255u << shift;
    remaining -= above;
    __syncwarp();
  }
  // the k-th key is `prefix`: take every key above it and the `remaining`
  // lowest-index keys equal to it
  uint32_t gt = 0, eq = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const bool in = base + i < n;
    gt += (in && key[i] > prefix) ? 1u : 0u;
    eq += (in && key[i] == prefix) ? 1u : 0u;
  }
  uint32_t eq_incl = eq;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, eq_incl, o);
    if (lane >= o) eq_incl += y;
  }
  const uint32_t eq_before = eq_incl - eq;
  const uint32_t take_eq = remaining > eq_before ? (remaining - eq_before < eq ? remaining - eq_before : eq) : 0u;
  const uint32_t sel = gt + take_eq;
  uint32_t sel_incl = sel;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, sel_incl, o);
    if (lane >= o) sel_incl += y;
  }
  uint32_t pos = sel_incl - sel, taken = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (base + i >= n) continue;
    const bool pick = key[i] > prefix || (key[i] == prefix && taken++ < take_eq);
    if (pick) {
      out[pos] = base + i;
      if (sout != nullptr) sout[pos] = __ldcg(srow + base + i);
      ++pos;
    }
  }
}

// ---------------------------------------------------------------------------
// prefill rows with bf16 keys: tcgen05 scoring, scores kept on chip
// ---------------------------------------------------------------------------
// One CTA owns kPfQ consecutive query rows of one sequence.  The MMA computes
// S^T = K Q^T with the entries as M (128 per tile, one per TMEM lane) and the
// (query, head) pairs as N (kPfQ * 4 = 128 columns), K = 64; an epilogue
// thread owns one entry of the tile and folds its 4 heads per query
// (s_q = sum_h relu(S[e, 4q+h]) w[q, h]) into the order-preserving 32-bit key
// of each query's score, which it stages in shared memory; eight epilogue
// warps work in two halves of 16 queries (64 accumulator columns) each, so
// every scheduler has two warps to interleave.  The keys are then read back
// query-major: eight consecutive lanes of a warp own one query and 16
// consecutive entries of the tile each, so a query's running state lives in
// registers of its own lanes and no two lanes of a warp share a histogram row
// unless they share the query; runs of equal bins are counted in a register
// before one atomic.  The exact top-k is a radix select on the key, in
// levels of 11, 11 and 10 bits, over passes that recompute the same scores (the MMA is
// cheap; no score leaves the SM):
//   passes 0-2: per-query 2048-bin histogram of key bits 31..21, then of bits
//               20..10 for entries whose top bits are the query's threshold
//               bin, then bits 9..0; a query whose threshold bin is taken
//               whole stops refining, and a pass scores only the queries that
//               still refine;
//   pass 3:     emission -- every entry above the threshold and the first
//               `need` entries equal to it, in ascending index order (ties
//               therefore go to the lower index), by a 4-lane scan per query.
// A pass no query needs only waits for its tiles.  The key tiles stream by TMA
// (128-byte swizzle, no multicast) through a ring of stages, one thread issues
// the MMAs into two TMEM buffers, and all waits are bounded.
constexpr int kPfQ = 32;         // query rows per CTA (x 4 heads = 128 MMA columns)
constexpr int kPfTile = 128;     // entries per tile (MMA M)
constexpr int kPfStages = 3;
constexpr int kPfThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue (two halves of 16 queries)
constexpr int kPfEpi = 256;      // epilogue threads
constexpr int kPfLanesQ = 8;     // lanes per query in the query-major phase (16 entries of a tile each)
constexpr int kPfLevels = 3;     // histogram levels: key bits 31..21, 20..10, 9..0
constexpr int kPfHistW = 1025;   // words per query histogram: 2048 16-bit bins + 1 pad (bank spread)
constexpr int kPfKeyW = 132;     // words per query row of staged keys: 4 quarters x 33 (bank spread)
__host__ __device__ constexpr int pf_level_bits(int level) { return level == 2 ? 10 : 11; }
__host__ __device__ constexpr int pf_level_shift(int level) { return level == 0 ? 21 : (level == 1 ? 10 : 0); }

struct PfLayout {
  static constexpr size_t kK = 0;                                  // [kPfStages][128 entries][128 B]
  static constexpr size_t kQ = kK + kPfStages * 16384;             // [128 (query, head)][128 B]
  static constexpr size_t kHist = kQ + 16384;                      // [kPfQ][kPfHistW] u32
  static constexpr size_t kKeys = kHist + kPfQ * kPfHistW * 4;     // [kPfQ][kPfKeyW] u32
  static constexpr size_t kW = kKeys + kPfQ * kPfKeyW * 4;         // [128] fp32
  static constexpr size_t kQs = kW + 128 * 4;                      // per-query state, 7 x [kPfQ] u32
  static constexpr size_t kBars = (kQs + 7 * kPfQ * 4 + 7) / 8 * 8;
  static constexpr size_t kTotal = kBars + 96 + 1024;              // + alignment slack
};
static_assert(PfLayout::kTotal <= 232448, "prefill indexer shared memory above the per-block limit");

struct PfParams {
  const __nv_bfloat16* qI;  // [B, Tq, 4, 64]
  const float* wI;          // [B, Tq, 4]
  int64_t Tq, N, q_pos0;
  int m, k;
  int64_t groups;           // CTAs: B * ceil(Tq / kPfQ), or an upper bound for packed sequences
  int32_t* idx;             // [B, Tq, k]
  // packed sequences (nullable): sequence s owns query rows [cu_tok[s], cu_tok[s+1])
  // (positions from 0) and key rows [cu_ent[s], cu_ent[s+1]) of a [1][total][64]
  // key tensor; CTA g is group g - cu_grp[s] of kPfQ rows of sequence s
  const int32_t* cu_tok;
  const int32_t* cu_ent;
  const int32_t* cu_grp;
  int n_seqs;
};

__global__ void __launch_bounds__(kPfThreads, 1) indexer_prefill_kernel(PfParams p,
                                                                        const __grid_constant__ CUtensorMap kmap) {
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* Kst = smem + PfLayout::kK;
  uint8_t* Qs = smem + PfLayout::kQ;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + PfLayout::kHist);
  uint32_t* keys_s = reinterpret_cast<uint32_t*>(smem + PfLayout::kKeys);
  float* w_s = reinterpret_cast<float*>(smem + PfLayout::kW);
  uint32_t* qs = reinterpret_cast<uint32_t*>(smem + PfLayout::kQs);
  uint32_t* nv_s = qs;                 // visible entries of query j
  uint32_t* level_s = qs + kPfQ;       // 0..3: refining at that level; kPfLevels: threshold known
  uint32_t* prefix_s = qs + 2 * kPfQ;  // key bytes fixed so far
  uint32_t* rem_s = qs + 3 * kPfQ;     // entries still to take at the current level
  uint32_t* shift_s = qs + 4 * kPfQ;   // emission: compare key >> shift with thr, take need ties
  uint32_t* thr_s = qs + 5 * kPfQ;
  uint32_t* need_s = qs + 6 * kPfQ;    // (7 state arrays)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + PfLayout::kBars);  // [kPfStages]
  uint64_t* empty = full + kPfStages;                                     // [kPfStages]
  uint64_t* tfull = empty + kPfStages;                                    // [2]
  uint64_t* tempty = tfull + 2;                                           // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t grp = p.groups - 1 - static_cast<int64_t>(blockIdx.x);  // late (long) rows first
  // this CTA's rows: global rows row0.., positions t0.., keys at tensor-map rows
  // key0.. of batch kb, Nseq of them
  int64_t row0, t0, key0, Nseq;
  int kb, nq;
  if (p.cu_tok != nullptr) {
    if (grp >= __ldg(p.cu_grp + p.n_seqs)) return;  // past the last group (the grid is an upper bound)
    const int sq = seq_of(p.cu_grp, p.n_seqs, grp);
    const int64_t len = __ldg(p.cu_tok + sq + 1) - __ldg(p.cu_tok + sq);
    t0 = (grp - __ldg(p.cu_grp + sq)) * kPfQ;
    row0 = __ldg(p.cu_tok + sq) + t0;
    nq = static_cast<int>((len - t0) < kPfQ ? (len - t0) : kPfQ);
    key0 = __ldg(p.cu_ent + sq);
    Nseq = __ldg(p.cu_ent + sq + 1) - key0;
    kb = 0;
  } else {
    const int64_t gpb = (p.Tq + kPfQ - 1) / kPfQ;
    const int64_t b = grp / gpb;
    const int64_t r0 = (grp % gpb) * kPfQ;
    nq = static_cast<int>((p.Tq - r0) < kPfQ ? (p.Tq - r0) : kPfQ);
    row0 = b * p.Tq + r0;
    t0 = p.q_pos0 + r0;
    key0 = 0;
    Nseq = p.N;
    kb = static_cast<int>(b);
  }
  const int64_t nv_max = visible(t0 + nq - 1, p.m, Nseq);
  const int k = p.k;

  if (tid < kPfQ) {
    const int j = tid;
    const uint32_t nv = j < nq ? static_cast<uint32_t>(visible(t0 + j, p.m, Nseq)) : 0u;
    nv_s[j] = nv;
    const bool partial = nv > static_cast<uint32_t>(k);
    level_s[j] = partial ? 0u : static_cast<uint32_t>(kPfLevels);
    prefix_s[j] = 0u;
    rem_s[j] = static_cast<uint32_t>(k);
    shift_s[j] = 0u;   // with thr 0 every visible key (>= 0x007fffff) is above: all visible entries
    thr_s[j] = 0u;
    need_s[j] = 0u;
  }
  if (nv_max <= k) {  // every row of the CTA keeps all its visible entries: no scoring at all
    __syncthreads();
    for (int i = tid; i < nq * k; i += kPfThreads) {
      const int j = i / k, c = i % k;
      p.idx[(row0 + j) * k + c] = c < static_cast<int>(nv_s[j]) ? c : -1;
    }
    return;
  }
  const int ntiles = static_cast<int>((nv_max + kPfTile - 1) / kPfTile);
  constexpr int kPasses = kPfLevels + 1;

  if (tid == 0) {
    for (int i = 0; i < kPfStages; ++i) {
      tc::bar_init(&full[i], 1);
      tc::bar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::bar_init(&tfull[i], 1);
      tc::bar_init(&tempty[i], kPfEpi);
    }
    tc::bar_init_fence();
  }
  if (warp == 1) tc::tmem_alloc(tslot, 256);
  // Q: row n = (query n/4, head n%4), 64 dims = 128 B, swizzled K-major; rows past nq are zero
  for (int piece = tid; piece < 128 * 8; piece += kPfThreads) {
    const int n = piece >> 3, ch = piece & 7;
    const bool ok = (n >> 2) < nq;
    cp_async16(Qs + tc::sw128(n, ch), ok ? p.qI + ((row0 + (n >> 2)) * kHI + (n & 3)) * kDI + ch * 8 : p.qI,
               ok ? 16 : 0);
  }
  cp_async_commit();
  if (tid < 128) w_s[tid] = (tid >> 2) < nq ? p.wI[(row0 + (tid >> 2)) * kHI + (tid & 3)] : 0.f;
  for (int i = tid; i < kPfQ * kPfHistW; i += kPfThreads) hist[i] = 0u;
  cp_async_wait<0>();
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;
  const int total = kPasses * ntiles;

  if (warp == 0) {
    // ===================== TMA producer: the same tiles, once per pass =====================
    if (lane == 0) {
      for (int it = 0; it < total; ++it) {
        const int st = it % kPfStages;
        if (it >= kPfStages && !tc::bar_wait(&empty[st], static_cast<uint32_t>(((it / kPfStages) - 1) & 1))) break;
        tc::bar_arrive_expect_tx(&full[st], 16384u);
        tc::tma_load_3d(Kst + st * 16384, &kmap, 0, static_cast<int>(key0 + (it % ntiles) * kPfTile), kb, &full[st]);
      }
    }
  } else if (warp == 1) {
    // ===================== MMA issue (one thread) =====================
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16(128, 128, false, false);
      const uint32_t qa = smem_u32(Qs);
      for (int it = 0; it < total; ++it) {
        const int st = it % kPfStages, buf = it & 1;
        if (it >= 2 && !tc::bar_wait(&tempty[buf], static_cast<uint32_t>(((it >> 1) - 1) & 1))) break;
        if (!tc::bar_wait(&full[st], static_cast<uint32_t>((it / kPfStages) & 1))) break;
        tc::fence_after_sync();
        const uint32_t ka = smem_u32(Kst + st * 16384);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc::mma_bf16_ss(tmem + static_cast<uint32_t>(buf * 128), tc::desc_sw128(ka + kk * 32, 16, 1024),
                          tc::desc_sw128(qa + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        tc::mma_commit(&empty[st]);
        tc::mma_commit(&tfull[buf]);
      }
    }
  } else {
    // ===================== epilogue =====================
    // scoring: thread = entry et of the tile (its TMEM lane), queries of half
    // hq; then query-major: thread = (query qj of the half, part qp: entries
    // 16 qp .. 16 qp + 15 of the tile)
    const int ew = warp - 2;            // 0..7
    const int hq = ew >> 2;             // query half: queries 16 hq .. 16 hq + 15
    const int q4 = warp & 3;            // TMEM lane quarter of this warp
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const int et = q4 * 32 + lane;      // entry within the tile (scoring)
    const int htid = (ew & 3) * 32 + lane;  // 0..127 within the half
    const int qj = hq * 16 + (htid >> 3), qp = htid & 7;
    const int64_t qrow = row0 + qj;
    const int bar_half = 3 + hq;        // named barrier of this half
    // key slot of entry e for query j: quarter-padded rows spread the banks
    auto key_slot = [&](int j, int e) { return j * kPfKeyW + (e >> 5) * 33 + (e & 31); };
    // A wait that runs out (recorded in the device error word) skips the later
    // waits but keeps the loop and its named barriers, so the warps stay in
    // step and the CTA finishes; its output is then not valid.
    bool healthy = true;
    int it = 0;
    uint32_t sel_done = 0u, ties_done = 0u;  // emission running totals of query qj (same in its 8 lanes)
    for (int pass = 0; pass < kPasses; ++pass) {
      const bool emit = pass == kPfLevels;
      // queries of this half that need their scores in this pass (bit j - 16 hq)
      uint32_t need_mask = 0u;
      for (int j = 0; j < 16; ++j) {
        const int jq = hq * 16 + j;
        const bool w = emit ? nv_s[jq] > 0u : level_s[jq] == static_cast<uint32_t>(pass);
        need_mask |= w ? (1u << j) : 0u;
      }
      // this thread's query state for the pass
      const uint32_t nv_q = nv_s[qj], pre_q = prefix_s[qj];
      const uint32_t sh_q = shift_s[qj], thr_q = thr_s[qj], need_q = need_s[qj];
      const bool mine = (need_mask >> (qj - hq * 16)) & 1u;
      for (int tile = 0; tile < ntiles; ++tile, ++it) {
        const int buf = it & 1;
        if (healthy) healthy = tc::bar_wait(&tfull[buf], static_cast<uint32_t>((it >> 1) & 1));
        tc::fence_after_sync();
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {  // 8 queries (32 accumulator columns) at a time
          const uint32_t cmask = (need_mask >> (c * 8)) & 0xffu;
          float v[32];
          if (cmask) tc::tmem_ld32(tmem + lane_base + static_cast<uint32_t>(buf * 128 + hq * 64 + c * 32), v);
          if (c == 1) {
            tc::fence_before_sync();
            bar_arrive(&tempty[buf]);
          }
          if (!cmask) continue;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {  // all 8 queries of the chunk (unneeded keys are not read)
            const int j = hq * 16 + c * 8 + jj;
            const float4 w4 = *reinterpret_cast<const float4*>(w_s + 4 * j);
            const float sc = fmaxf(v[4 * jj], 0.f) * w4.x + fmaxf(v[4 * jj + 1], 0.f) * w4.y +
                             fmaxf(v[4 * jj + 2], 0.f) * w4.z + fmaxf(v[4 * jj + 3], 0.f) * w4.w;
            keys_s[key_slot(j, et)] = f2key(sc + 0.0f);
          }
        }
        if (!need_mask) continue;        // uniform for the half
        named_sync_ix(bar_half, 128);    // this half's keys of the tile are staged
        if (mine) {
          const int e0 = qp * 16;                                  // this thread's first entry of the tile
          const uint32_t eabs0 = static_cast<uint32_t>(tile * kPfTile + e0);
          const int nvis = static_cast<int>(nv_q > eabs0 ? (nv_q - eabs0 < 16u ? nv_q - eabs0 : 16u) : 0u);
          uint32_t kv[16];
          {
            const uint32_t* kr = keys_s + key_slot(qj, e0);  // 16 consecutive slots in one quarter
#pragma unroll
            for (int i = 0; i < 16; ++i) kv[i] = kr[i];
          }
          if (!emit) {
            const int bsh = pf_level_shift(pass);
            const uint32_t bmask = (1u << pf_level_bits(pass)) - 1u;
            const int psh = bsh + pf_level_bits(pass);  // bits above this level's
            uint32_t* h = hist + qj * kPfHistW;
            uint32_t cur = 0xffffffffu, run = 0u;  // runs of equal bins: one atomic per run
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint32_t key = kv[i];
              const bool in = i < nvis && (pass == 0 || (key >> psh) == pre_q);
              const uint32_t bin = (key >> bsh) & bmask;
              if (in && bin != cur) {
                if (run) atomicAdd(h + (cur >> 1), run << ((cur & 1u) * 16));
                cur = bin;
                run = 0u;
              }
              run += in ? 1u : 0u;
            }
            if (run) atomicAdd(h + (cur >> 1), run << ((cur & 1u) * 16));
          }
        }
        if (emit) {  // every lane of the half: the scans below are warp-wide
          uint32_t gt = 0u, eq = 0u;
          const int e0 = qp * 16;
          const uint32_t eabs0 = static_cast<uint32_t>(tile * kPfTile + e0);
          if (mine) {
            const int nvis = static_cast<int>(nv_q > eabs0 ? (nv_q - eabs0 < 16u ? nv_q - eabs0 : 16u) : 0u);
            const uint32_t* kr = keys_s + key_slot(qj, e0);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint32_t kk = kr[i] >> sh_q;
              gt |= (i < nvis && kk > thr_q) ? (1u << i) : 0u;
              eq |= (i < nvis && kk == thr_q) ? (1u << i) : 0u;
            }
          }
          const uint32_t n_eq = __popc(eq);
          uint32_t tie_incl = n_eq;  // scan over the query's 8 lanes (entries in order)
#pragma unroll
          for (int o = 1; o < kPfLanesQ; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, tie_incl, o, kPfLanesQ);
            if (qp >= o) tie_incl += t;
          }
          const uint32_t tie0 = ties_done + tie_incl - n_eq;  // rank of this thread's first tie
          const uint32_t take = need_q > tie0 ? (need_q - tie0 < n_eq ? need_q - tie0 : n_eq) : 0u;
          // the first `take` tie bits (lowest entries) are selected
          uint32_t eq_sel = eq;
          for (uint32_t drop = n_eq - take; drop > 0; --drop) eq_sel &= ~(0x80000000u >> __clz(eq_sel));
          const uint32_t sel = gt | eq_sel;
          const uint32_t n_sel = __popc(sel);
          uint32_t sel_incl = n_sel;
#pragma unroll
          for (int o = 1; o < kPfLanesQ; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, sel_incl, o, kPfLanesQ);
            if (qp >= o) sel_incl += t;
          }
          uint32_t pos = sel_done + sel_incl - n_sel;
          for (uint32_t m = sel; m != 0u; m &= m - 1u) {
            if (pos < static_cast<uint32_t>(k)) p.idx[qrow * k + pos] = static_cast<int32_t>(eabs0 + __ffs(m) - 1);
            ++pos;
          }
          const int last = (lane & ~(kPfLanesQ - 1)) | (kPfLanesQ - 1);
          ties_done += __shfl_sync(0xffffffffu, tie_incl, last);
          sel_done += __shfl_sync(0xffffffffu, sel_incl, last);
        }
        named_sync_ix(bar_half, 128);  // the keys are read: the next tile may overwrite them
      }
      if (emit) break;
      // ---- thresholds of the queries that refined at this level (all 8 warps) ----
      named_sync_ix(2, kPfEpi);
      const int nbits = pf_level_bits(pass);
      const int per_lane = (1 << nbits) / 32;  // bins per lane, walked from the top
      for (int j = ew; j < kPfQ; j += 8) {
        if (level_s[j] != static_cast<uint32_t>(pass)) continue;  // uniform in the warp
        const uint32_t* h = hist + j * kPfHistW;
        const int top = (1 << nbits) - lane * per_lane;  // this lane's bins [top - per_lane, top)
        // the lanes' bin sums, read transposed: at step c the warp reads lane c's words side by side
        // (consecutive words, no bank conflict) and reduces them, and lane c keeps the total
        const int wpl = per_lane / 2;  // words per lane
        uint32_t sum = 0;
        for (int c = 0; c < 32; ++c) {
          const int wbase = ((1 << nbits) - (c + 1) * per_lane) / 2;
          uint32_t v = lane < wpl ? h[wbase + lane] : 0u;
          v = (v & 0xffffu) + (v >> 16);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == c) sum = v;
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        const uint32_t excl = incl - sum;
        const uint32_t rem = rem_s[j];
        if (excl < rem && incl >= rem) {
          uint32_t acc = excl;
          for (int bb = top - 1; bb >= top - per_lane; --bb) {
            const uint32_t cb = (h[bb >> 1] >> ((bb & 1) * 16)) & 0xffffu;
            if (acc + cb >= rem) {
              const uint32_t nrem = rem - acc;  // still needed from bin bb
              const uint32_t pref = (prefix_s[j] << nbits) | static_cast<uint32_t>(bb);
              if (cb == nrem || pass == kPfLevels - 1) {  // threshold found; its ties go in index order
                shift_s[j] = static_cast<uint32_t>(pf_level_shift(pass));
                thr_s[j] = pref;
                need_s[j] = nrem;
                level_s[j] = static_cast<uint32_t>(kPfLevels);
              } else {
                prefix_s[j] = pref;
                rem_s[j] = nrem;
                level_s[j] = static_cast<uint32_t>(pass + 1);
              }
              break;
            }
            acc += cb;
          }
        }
      }
      named_sync_ix(2, kPfEpi);  // every warp is done reading the histograms
      for (int i = ew * 32 + lane; i < kPfQ * kPfHistW; i += kPfEpi) hist[i] = 0u;
      named_sync_ix(2, kPfEpi);
    }
    // padding after each query's selection (its 8 lanes hold the running total)
    if (qj < nq) {
      const uint32_t done = sel_done < static_cast<uint32_t>(k) ? sel_done : static_cast<uint32_t>(k);
      for (uint32_t c = done + qp; c < static_cast<uint32_t>(k); c += kPfLanesQ) p.idx[qrow * k + c] = -1;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// long-row path: histogram fused into scoring, then two select kernels.  The
// first classifies every entry against the row's threshold bin (bitmap words
// for the entries above it, a candidate list of the entries in it, a count of
// the entries above it per chunk).  The second resolves the cut inside the
// bin and writes the ascending list: every CTA its own span of the row, at the
// offset of the selected entries before the span.
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 512;
constexpr int kSelChunk = 8192;                 // entries per classifying CTA
constexpr int kCandSmem = 4096;                 // threshold-bin candidates kept in shared memory
#ifndef CSA_EMIT_THREADS
#define CSA_EMIT_THREADS 512
#endif
#ifndef CSA_EMIT_WPT
#define CSA_EMIT_WPT 2
#endif
constexpr int kEmitThreads = CSA_EMIT_THREADS;
constexpr int kEmitWpt = CSA_EMIT_WPT;                // consecutive bitmap words per thread
constexpr int kEmitWords = kEmitWpt * kEmitThreads;  // bitmap words per emitting CTA
constexpr int kEmitSpan = 32 * kEmitWords;      // entries per emitting CTA
static_assert(kEmitSpan % kSelChunk == 0, "an emitting span covers whole classifying chunks");

struct LongWs {
  float* scores;        // [R, pitch] (pitch = N rounded up to 4: 16-byte aligned rows)
  uint32_t* hist;       // [R, kHistBins]    (zeroed per call)
  uint32_t* cand_cnt;   // [R]               (zeroed per call)
  int2* rinfo;          // [R]: (threshold bin, entries still needed from it)
  uint32_t* ccnt;       // [R, nch]: entries above the threshold bin, per chunk
  uint2* cand;          // [R, N]: (key, index) of the threshold bin's entries
  uint32_t* bitmap;     // [R, W]: bit e set when entry e lies above the threshold bin
  int64_t W;
  int64_t pitch;
  int64_t nch;          // chunks per row, ceil(N / kSelChunk)
};

// Per CTA (one chunk of a row): the row's threshold bin from its complete
// histogram (every CTA of the row derives it, its score loads already in
// flight), then a bitmap word for every 32 entries (entries above the
// threshold bin), the chunk's count of such entries, and the threshold bin's
// entries appended to the row's candidate list (gathered in shared memory
// first, one global atomic per CTA).  Rows with no more visible entries than
// k are written here whole.
__global__ void __launch_bounds__(kSelThreads, 2) topk_classify_kernel(LongWs ws, int64_t N, int64_t Tq,
                                                                       int64_t q_pos0, int m, int k,
                                                                       int32_t* __restrict__ idx,
                                                                       float* __restrict__ scores_out) {
  pdl_wait();
  extern __shared__ __align__(16) uint8_t sel_smem[];  // candidates of the chunk
  uint2* cand_s = reinterpret_cast<uint2*>(sel_smem);
  __shared__ uint32_t n_cand, n_above, base_s;
  __shared__ int32_t thr_s[2];
  __shared__ uint32_t scan_sh[32];
  const int64_t row = blockIdx.y;
  const int64_t nv = visible(q_pos0 + row % Tq, m, N);
  const int64_t e_begin = static_cast<int64_t>(blockIdx.x) * kSelChunk;
  int32_t* out = idx + row * k;
  float* sout = scores_out != nullptr ? scores_out + row * k : nullptr;
  const float* srow = ws.scores + row * ws.pitch;
  if (nv == 0) {  // no entry visible yet (the scoring kernel skipped the row): all padding
    if (blockIdx.x == 0) write_prefix_ids(out, 0, k, sout, srow);
    return;
  }
  if (e_begin >= nv) return;
  if (nv <= k) {  // every visible entry is selected
    if (blockIdx.x == 0) write_prefix_ids(out, nv, k, sout, srow);
    return;
  }
  const int64_t e_end = (e_begin + kSelChunk) < nv ? (e_begin + kSelChunk) : nv;
  const int lane = threadIdx.x & 31;
  // warp w scans entries [e_begin + 512 w, e_begin + 512 (w + 1)), four per
  // lane per step (16-byte loads; rows are 16-byte aligned and padded)
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
  // the threshold bin and the count still needed from it (nv > k: a bin exists)
  row_threshold<kSelThreads>(ws.hist + row * kHistBins, nv, k, thr_s, scan_sh);
  if (threadIdx.x == 0) {
    n_cand = 0;
    n_above = 0;
  }
  __syncthreads();
  const uint32_t tb = static_cast<uint32_t>(thr_s[0]);
  uint32_t n_up = 0;  // entries above the threshold bin seen by this lane
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
    n_up += __popc(above);
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
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n_up += __shfl_xor_sync(0xffffffffu, n_up, o);
  if (lane == 0 && n_up) atomicAdd(&n_above, n_up);
  __syncthreads();
  const uint32_t nc = n_cand < static_cast<uint32_t>(kCandSmem) ? n_cand : static_cast<uint32_t>(kCandSmem);
  if (threadIdx.x == 0) {
    if (nc) base_s = atomicAdd(ws.cand_cnt + row, nc);
    ws.ccnt[row * ws.nch + blockIdx.x] = n_above;
    if (blockIdx.x == 0) ws.rinfo[row] = make_int2(thr_s[0], thr_s[1]);
  }
  pdl_trigger();  // the emitting kernel may be scheduled while the candidates are stored
  __syncthreads();
  for (uint32_t c = threadIdx.x; c < nc; c += kSelThreads) ws.cand[row * N + base_s + c] = cand_s[c];
}

// Per CTA (one span of kEmitSpan entries of a row whose visible entries
// outnumber k): radix-selects the `need` best threshold-bin candidates on the
// composite key (score key << 32 | ~index, so equal scores go to the lower
// index), the same cut in every CTA of the row; sets the selected candidates
// of its span in the span's bitmap words; and writes the span's selected
// entries in ascending order at the offset of those before it (the above-bin
// counts of the earlier chunks plus the selected candidates before the span).
__global__ void __launch_bounds__(kEmitThreads, 1) topk_emit_kernel(LongWs ws, int64_t N, int64_t Tq,
                                                                    int64_t q_pos0, int m, int k,
                                                                    int32_t* __restrict__ idx,
                                                                    float* __restrict__ scores_out) {
  pdl_wait();
  extern __shared__ __align__(16) uint8_t emit_smem[];
  uint2* cand_s = reinterpret_cast<uint2*>(emit_smem);                                  // [kCandSmem]
  uint32_t* wsm = reinterpret_cast<uint32_t*>(emit_smem + kCandSmem * sizeof(uint2));  // [kEmitWords]
  __shared__ uint32_t hist[256];
  __shared__ uint32_t dig[3];
  __shared__ uint32_t before_s;  // selected entries before the span
  __shared__ uint32_t scan_sh[32];
  const int64_t row = blockIdx.y;
  const int64_t nv = visible(q_pos0 + row % Tq, m, N);
  if (nv <= k) return;  // the classifying kernel wrote the whole list
  const int64_t e_begin = static_cast<int64_t>(blockIdx.x) * kEmitSpan;
  if (e_begin >= nv) return;
  const int64_t e_end = (e_begin + kEmitSpan) < nv ? (e_begin + kEmitSpan) : nv;
  const int64_t words = (nv + 31) >> 5;
  const int64_t w_begin = e_begin >> 5;
  const int tid = threadIdx.x, lane = tid & 31;
  int32_t* out = idx + row * k;
  float* sout = scores_out != nullptr ? scores_out + row * k : nullptr;
  const float* srow = ws.scores + row * ws.pitch;
  const uint32_t* gbm = ws.bitmap + row * ws.W;

  // ---- loads in flight together: the span's bitmap words, the candidates
  // (when they fit in shared memory), the above-bin counts of earlier chunks
  const uint32_t cnt = __ldcg(ws.cand_cnt + row);
  const int2 ri = __ldcg(ws.rinfo + row);
  const uint2* cand = ws.cand + row * N;
  const bool cand_in_smem = cnt <= static_cast<uint32_t>(kCandSmem);
  uint32_t wv[kEmitWpt];
#pragma unroll
  for (int u = 0; u < kEmitWpt; ++u) {
    const int64_t wi = w_begin + kEmitWpt * tid + u;
    wv[u] = wi < words ? __ldcg(gbm + wi) : 0u;
  }
  constexpr int kCandPerThread = kCandSmem / kEmitThreads;
  uint2 cv[kCandPerThread];
  if (cand_in_smem) {
#pragma unroll
    for (int u = 0; u < kCandPerThread; ++u) {
      const uint32_t c = u * kEmitThreads + tid;
      cv[u] = c < cnt ? __ldcg(cand + c) : make_uint2(0, 0);
    }
  }
  const int64_t chunks_before = e_begin / kSelChunk;
  uint32_t before = 0;
  for (int64_t c = tid; c < chunks_before; c += kEmitThreads) before += __ldcg(ws.ccnt + row * ws.nch + c);
  if (tid == 0) before_s = 0;
#pragma unroll
  for (int u = 0; u < kEmitWpt; ++u) wsm[kEmitWpt * tid + u] = wv[u];
  if (cand_in_smem) {
#pragma unroll
    for (int u = 0; u < kCandPerThread; ++u) {
      const uint32_t c = u * kEmitThreads + tid;
      if (c < cnt) cand_s[c] = cv[u];
    }
    cand = cand_s;
  }
  __syncthreads();

  // ---- the cut inside the threshold bin: radix select on the 52 low composite bits
  uint32_t remaining = static_cast<uint32_t>(ri.y);
  uint64_t prefix = static_cast<uint64_t>(static_cast<uint32_t>(ri.x)) << 52;
  uint64_t mask = 0xfffull << 52;
  uint32_t in_bucket = cnt;
  for (int pass = 0; pass < 7 && in_bucket != remaining; ++pass) {
    const int sh = pass < 6 ? 44 - 8 * pass : 0;
    const uint64_t dmask = pass < 6 ? 255ull : 15ull;
    for (int j = tid; j < 256; j += kEmitThreads) hist[j] = 0;
    __syncthreads();
    for (uint32_t c = tid; c < cnt; c += kEmitThreads) {
      const uint2 kv = cand_in_smem ? cand[c] : __ldcg(cand + c);
      const uint64_t x = (static_cast<uint64_t>(kv.x) << 32) | (0xffffffffu - kv.y);
      if ((x & mask) == prefix) atomicAdd(&hist[(x >> sh) & dmask], 1u);
    }
    __syncthreads();
    if (tid < 32) find_digit_256(hist, remaining, dig);
    __syncthreads();
    prefix |= static_cast<uint64_t>(dig[0]) << sh;
    mask |= dmask << sh;
    remaining -= dig[1];
    in_bucket = dig[2];
    __syncthreads();
  }
  // ---- selected candidates: counted before the span, set in its words inside it
  for (uint32_t c = tid; c < cnt; c += kEmitThreads) {
    const uint2 kv = cand_in_smem ? cand[c] : __ldcg(cand + c);
    const uint64_t x = (static_cast<uint64_t>(kv.x) << 32) | (0xffffffffu - kv.y);
    if ((x & mask) >= prefix) {
      if (static_cast<int64_t>(kv.y) < e_begin) {
        ++before;
      } else if (static_cast<int64_t>(kv.y) < e_end) {
        atomicOr(&wsm[(kv.y >> 5) - w_begin], 1u << (kv.y & 31));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
  if (lane == 0 && before) atomicAdd(&before_s, before);
  __syncthreads();

  // ---- ascending emission: thread t owns words [t, t + 1) * kEmitWpt of the span
  uint32_t nbits = 0;
#pragma unroll
  for (int u = 0; u < kEmitWpt; ++u) {
    wv[u] = wsm[kEmitWpt * tid + u];
    nbits += __popc(wv[u]);
  }
  uint32_t total;
  uint32_t p = before_s + block_excl_scan(nbits, &total, scan_sh);
  const int64_t e0 = (w_begin + kEmitWpt * tid) << 5;
#pragma unroll
  for (int u = 0; u < kEmitWpt; ++u) {
    uint32_t word = wv[u];
    while (word) {
      const int bit = __ffs(word) - 1;
      word &= word - 1;
      if (p < static_cast<uint32_t>(k)) {
        const int64_t e = e0 + 32 * u + bit;
        out[p] = static_cast<int32_t>(e);
        if (sout != nullptr) sout[p] = __ldcg(srow + e);
      }
      ++p;
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool use_row_path(int64_t R, int64_t N) { return N <= kRowPathMaxN && R > 256; }
// Prefill rows with bf16 keys run the on-chip tcgen05 kernel (16-bit
// histogram bins: up to 65535 entries) when its 32-row CTAs fill the device
// at least once; fewer rows (under 32 per SM) take the row path, whose
// per-row select runs one CTA per row (2048 rows of the 2048-token prefill:
// 54 µs against 78 µs on chip, measured).
constexpr int64_t kPrefillTcMaxN = 65535;
bool use_prefill_tc(int64_t R, int64_t N) { return N <= kPrefillTcMaxN && R >= 32LL * num_sms(); }

struct LongLayout {
  size_t scores, hist, cnt, zero_end, rinfo, ccnt, cand, bitmap, total;
  int64_t W, pitch, nch;
};

LongLayout long_layout(int64_t R, int64_t N) {
  LongLayout L;
  L.W = ((N + 31) / 32 + 15) / 16 * 16;  // 16-word multiple: vector reads stay in the row
  L.pitch = (N + 3) / 4 * 4;
  L.nch = (N + kSelChunk - 1) / kSelChunk;
  size_t off = 0;
  L.scores = off; off = align_up(off + static_cast<size_t>(R) * L.pitch * 4);
  L.hist = off;   off += static_cast<size_t>(R) * kHistBins * 4;     // hist and cnt: zeroed together
  L.cnt = off;    off += static_cast<size_t>(R) * 4;
  L.zero_end = off;
  off = align_up(off);
  L.rinfo = off;  off = align_up(off + static_cast<size_t>(R) * 8);
  L.ccnt = off;   off = align_up(off + static_cast<size_t>(R) * L.nch * 4);
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

// Workspace of the bf16-key call (coded = false) or of the E4M3 / E2M1 calls.
// Prefill rows with bf16 keys keep their scores on chip and need none.
size_t workspace_bytes(int64_t B, int64_t Tq, int64_t N, bool coded = false) {
  const int64_t R = query_rows(B, Tq);
  if (R <= 0 || N <= 0 || N >= (int64_t(1) << 31)) return 0;
  if (!coded && use_prefill_tc(R, N)) return 0;
  if (coded && use_row_path(R, N)) return align_up(static_cast<size_t>(R) * N * 4);
  return long_layout(R, N).total;
}

}  // namespace
}  // namespace csa

namespace csa {
// Reads (and optionally clears) this unit's device error word.
CSA_DEFINE_DEVICE_ERROR_READER(indexer_device_error)
}  // namespace csa

extern "C" {

size_t csa_indexer_topk_workspace_size(int64_t B, int64_t Tq, int64_t N, int32_t k) {
  (void)k;
  if (B < 0 || Tq < 0 || N < 0) return 0;
  return csa::workspace_bytes(B, Tq, N, false);
}

size_t csa_indexer_topk_coded_workspace_size(int64_t B, int64_t Tq, int64_t N, int32_t k) {
  (void)k;
  if (B < 0 || Tq < 0 || N < 0) return 0;
  return csa::workspace_bytes(B, Tq, N, true);
}

}  // extern "C"

namespace csa {
namespace {
constexpr int kRowGroup = 8;  // query rows per scoring CTA on the row path

__global__ void fill_kernel(float* __restrict__ dst, int64_t n, float v) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = v;
}

// Scoring kernel over `groups` groups of query rows, then one top-k CTA per row.
csa_status launch_row_path(const char* name, ScoreParams& p, const RowsParams& rp, int64_t groups, int64_t R,
                           int64_t max_n, int kf, cudaStream_t s) {
  p.chunk = 2048;
  dim3 grid(static_cast<unsigned>((max_n + p.chunk - 1) / p.chunk), static_cast<unsigned>(groups));
  const dim3 block(kScoreThreads);
  prof_begin(s);
  const cudaError_t e =
      kf == kKeyE4M3   ? launch_pdl(score_kernel<kRowGroup, kKeyE4M3>, grid, block, score_tile_bytes(kf), s, 1, p)
      : kf == kKeyE2M1 ? launch_pdl(score_kernel<kRowGroup, kKeyE2M1>, grid, block, score_tile_bytes(kf), s, 1, p)
                       : launch_pdl(score_kernel<kRowGroup, kKeyBF16>, grid, block, score_tile_bytes(kf), s, 1, p);
  prof_end(s);
  if (csa_status st = check_launch(name, e); st != CSA_OK) return st;
  if (max_n <= kWarpRowMaxN)  // short rows: one warp per row
    return check_launch(name, launch_pdl(topk_rows_warp_kernel, dim3(static_cast<unsigned>((R + 7) / 8)), dim3(256),
                                         0, s, 1, rp, R));
  const size_t smem = static_cast<size_t>(max_n) * 4;
  if (!ensure_smem(reinterpret_cast<const void*>(topk_rows_kernel), kRowPathMaxN * 4))
    return fail(CSA_ERR_CUDA, "%s: cannot raise shared memory limit", name);
  return check_launch(name, launch_pdl(topk_rows_kernel, dim3(static_cast<unsigned>(R)), dim3(1024), smem, s, 1, rp));
}

// Offsets of each packed sequence's first group of `gsize` query rows.
__global__ void __launch_bounds__(1024) group_table_kernel(const int32_t* __restrict__ cu_tok, int n, int gsize,
                                                           int32_t* __restrict__ cu_grp) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t scan_sh[32];
  uint32_t carry = 0;
  if (threadIdx.x == 0) cu_grp[0] = 0;
  for (int base = 0; base < n; base += 1024) {
    const int sq = base + static_cast<int>(threadIdx.x);
    const uint32_t v = sq < n ? static_cast<uint32_t>(cu_tok[sq + 1] - cu_tok[sq] + gsize - 1) / gsize : 0u;
    uint32_t total;
    const uint32_t ex = block_excl_scan(v, &total, scan_sh);
    if (sq < n) cu_grp[sq + 1] = static_cast<int32_t>(carry + ex + v);
    carry += total;
  }
}

csa_status encode_key_map(CUtensorMap* kmap, const void* kIc, int64_t B, int64_t N, const char* name) {
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return fail(CSA_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", name);
  CSA_REQUIRE(aligned16(kIc), "%s: kIc must be 16-byte aligned", name);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDI), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDI) * 2, static_cast<cuuint64_t>(N) * kDI * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kDI), 128u, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = encode(kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kIc), dims, strides, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA_ERR_CUDA, "%s: tensor map encoding failed (%d)", name, int(r));
  return CSA_OK;
}

csa_status launch_prefill_tc(const void* qI, const float* wI, const void* kIc, int64_t B, int64_t Tq, int64_t N,
                             int64_t q_pos0, int32_t m, int32_t k, int32_t* idx, cudaStream_t s,
                             const csa_packed* pk = nullptr, const int32_t* cu_grp = nullptr) {
  CUtensorMap kmap;
  memset(&kmap, 0, sizeof(kmap));
  // packed sequences: one [1][total_entries][64] key tensor
  if (csa_status st = encode_key_map(&kmap, kIc, pk ? 1 : B, pk ? pk->total_entries : N, "csa_indexer_topk");
      st != CSA_OK)
    return st;
  PfParams p;
  p.qI = static_cast<const __nv_bfloat16*>(qI);
  p.wI = wI;
  p.Tq = Tq;
  p.N = N;
  p.q_pos0 = q_pos0;
  p.m = m;
  p.k = k;
  p.groups = pk ? (pk->total_tokens / kPfQ + pk->n_seqs) : B * ((Tq + kPfQ - 1) / kPfQ);
  p.idx = idx;
  p.cu_tok = pk ? pk->cu_tokens : nullptr;
  p.cu_ent = pk ? pk->cu_entries : nullptr;
  p.cu_grp = cu_grp;
  p.n_seqs = pk ? pk->n_seqs : 0;
  if (!ensure_smem(reinterpret_cast<const void*>(indexer_prefill_kernel), static_cast<int>(PfLayout::kTotal)))
    return fail(CSA_ERR_CUDA, "csa_indexer_topk: cannot raise the shared memory limit");
  prof_begin(s);
  const cudaError_t e = launch_pdl(indexer_prefill_kernel, dim3(static_cast<unsigned>(p.groups)), dim3(kPfThreads),
                                   PfLayout::kTotal, s, 1, p, kmap);
  prof_end(s);
  return check_launch("csa_indexer_topk (prefill, tcgen05)", e);
}

struct PackedLayout {
  size_t scores, grp, total;
  int64_t pitch;
};
// The packed path keeps its scores on chip: the workspace holds only the
// per-sequence group table.
PackedLayout packed_layout(const csa_packed* pk, int32_t m) {
  PackedLayout L;
  L.pitch = ((static_cast<int64_t>(pk->max_tokens) + m - 1) / m + 3) / 4 * 4;
  L.scores = 0;
  L.grp = 0;
  L.total = align_up((static_cast<size_t>(pk->n_seqs) + 1) * 4);
  return L;
}

csa_status indexer_impl(const void* qI, const float* wI, const void* kIc, const uint8_t* kcodes, const float* kscale,
                        int64_t B, int64_t Tq, int64_t N, int64_t q_pos0, int32_t m, int32_t k, int32_t* idx,
                        void* workspace, size_t workspace_bytes, void* stream, float* scores_out = nullptr,
                        int kf = kKeyBF16) {
  clear_error();
  const bool e4 = kcodes != nullptr;  // coded keys (kf: E4M3 or E2M1)
  if (!e4) kf = kKeyBF16;
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
    if (scores_out != nullptr)
      return check_launch("csa_indexer_topk", launch_pdl(fill_kernel, dim3(static_cast<unsigned>((R * k + 255) / 256)),
                                                         dim3(256), 0, s, 1, scores_out, R * k, -INFINITY));
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
  const bool tc_rows = !e4 && scores_out == nullptr && use_prefill_tc(R, N);  // tcgen05 prefill path
  const size_t need = tc_rows ? 0 : csa::workspace_bytes(B, Tq, N, true);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(CSA_ERR_WORKSPACE, "csa_indexer_topk: workspace of %zu bytes needed (got %zu)", need,
                workspace_bytes);
  CSA_REQUIRE(need == 0 || aligned16(workspace), "csa_indexer_topk: workspace is not 16-byte aligned");
  if (tc_rows) return launch_prefill_tc(qI, wI, kIc, B, Tq, N, q_pos0, m, k, idx, s);

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
  p.pitch = N;
  p.cu_tok = p.cu_ent = p.cu_grp = nullptr;
  p.n_seqs = 0;
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  if (use_row_path(R, N)) {
    constexpr int QR = kRowGroup;
    p.scores = reinterpret_cast<float*>(ws);
    p.hist = nullptr;
    p.done = nullptr;
    p.thr = nullptr;
    p.k = k;
    const int64_t groups = (Tq + QR - 1) / QR;
    CSA_REQUIRE(B * groups < 65536, "csa_indexer_topk: too many query rows for one launch");
    RowsParams rp{p.scores, N, N, Tq, q_pos0, m, k, idx, nullptr, nullptr, 0, scores_out};
    return launch_row_path("csa_indexer_topk", p, rp, B * groups, R, N, kf, s);
  }

  const LongLayout L = long_layout(R, N);
  LongWs w;
  w.scores = reinterpret_cast<float*>(ws + L.scores);
  w.hist = reinterpret_cast<uint32_t*>(ws + L.hist);
  w.cand_cnt = reinterpret_cast<uint32_t*>(ws + L.cnt);
  w.rinfo = reinterpret_cast<int2*>(ws + L.rinfo);
  w.ccnt = reinterpret_cast<uint32_t*>(ws + L.ccnt);
  w.cand = reinterpret_cast<uint2*>(ws + L.cand);
  w.bitmap = reinterpret_cast<uint32_t*>(ws + L.bitmap);
  w.W = L.W;
  w.pitch = L.pitch;
  w.nch = L.nch;
  if (cudaMemsetAsync(w.hist, 0, L.zero_end - L.hist, s) != cudaSuccess)
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
  const void* skern = kf == kKeyE4M3   ? reinterpret_cast<const void*>(score_long_kernel<kKeyE4M3>)
                      : kf == kKeyE2M1 ? reinterpret_cast<const void*>(score_long_kernel<kKeyE2M1>)
                                       : reinterpret_cast<const void*>(score_long_kernel<kKeyBF16>);
  const size_t ssmem = kf == kKeyE4M3   ? LongShape<kKeyE4M3>::kSmem
                       : kf == kKeyE2M1 ? LongShape<kKeyE2M1>::kSmem
                                        : LongShape<kKeyBF16>::kSmem;
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
  const dim3 lblock(kLongThreads);
  const cudaError_t e = kf == kKeyE4M3   ? launch_pdl(score_long_kernel<kKeyE4M3>, grid, lblock, ssmem, s, 1, lp, kmap)
                        : kf == kKeyE2M1 ? launch_pdl(score_long_kernel<kKeyE2M1>, grid, lblock, ssmem, s, 1, lp, kmap)
                                         : launch_pdl(score_long_kernel<kKeyBF16>, grid, lblock, ssmem, s, 1, lp, kmap);
  prof_end(s);
  if (csa_status st = check_launch("indexer score (long rows)", e); st != CSA_OK) return st;
  const dim3 cgrid(static_cast<unsigned>(L.nch), static_cast<unsigned>(R));
  constexpr int kClassifySmem = kCandSmem * 8;
  constexpr int kEmitSmem = kCandSmem * 8 + kEmitWords * 4;
  if (!ensure_smem(reinterpret_cast<const void*>(topk_classify_kernel), kClassifySmem) ||
      !ensure_smem(reinterpret_cast<const void*>(topk_emit_kernel), kEmitSmem))
    return fail(CSA_ERR_CUDA, "csa_indexer_topk: cannot raise shared memory limit");
  if (csa_status st = check_launch("indexer classify",
                                   launch_pdl(topk_classify_kernel, cgrid, dim3(kSelThreads), kClassifySmem, s, 1, w, N,
                                              Tq, q_pos0, m, k, idx, scores_out));
      st != CSA_OK)
    return st;
  const dim3 egrid(static_cast<unsigned>((N + kEmitSpan - 1) / kEmitSpan), static_cast<unsigned>(R));
  return check_launch("indexer emit", launch_pdl(topk_emit_kernel, egrid, dim3(kEmitThreads), kEmitSmem, s, 1, w, N,
                                                 Tq, q_pos0, m, k, idx, scores_out));
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

csa_status csa_indexer_topk_with_scores(const void* qI, const float* wI, const void* kIc, int64_t B, int64_t Tq,
                                        int64_t N, int64_t q_pos0, int32_t m, int32_t k, int32_t* idx, float* scores,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  if (scores == nullptr || (reinterpret_cast<uintptr_t>(scores) & 3u))
    return csa::fail(CSA_ERR_INVALID_ARG, "csa_indexer_topk_with_scores: scores NULL or misaligned");
  return csa::indexer_impl(qI, wI, kIc, nullptr, nullptr, B, Tq, N, q_pos0, m, k, idx, workspace, workspace_bytes,
                           stream, scores);
}

csa_status csa_indexer_topk_e4m3(const void* qI, const float* wI, const uint8_t* kI_codes, const float* kI_scale,
                                 int64_t B, int64_t Tq, int64_t N, int64_t q_pos0, int32_t m, int32_t k, int32_t* idx,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  return csa::indexer_impl(qI, wI, nullptr, kI_codes, kI_scale, B, Tq, N, q_pos0, m, k, idx, workspace,
                           workspace_bytes, stream, nullptr, csa::kKeyE4M3);
}

csa_status csa_indexer_topk_e2m1(const void* qI, const float* wI, const uint8_t* kI_codes, const float* kI_scale,
                                 int64_t B, int64_t Tq, int64_t N, int64_t q_pos0, int32_t m, int32_t k, int32_t* idx,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  return csa::indexer_impl(qI, wI, nullptr, kI_codes, kI_scale, B, Tq, N, q_pos0, m, k, idx, workspace,
                           workspace_bytes, stream, nullptr, csa::kKeyE2M1);
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

extern "C" size_t csa_indexer_topk_packed_workspace_size(const csa_packed* packed, int32_t m, int32_t k) {
  (void)k;
  if (packed == nullptr || m < 1 || packed->n_seqs <= 0 || packed->max_tokens < 0 || packed->total_tokens <= 0 ||
      packed->total_tokens >= (int64_t(1) << 31))
    return 0;
  return csa::packed_layout(packed, m).total;
}

extern "C" csa_status csa_indexer_topk_packed(const void* qI, const float* wI, const void* kIc,
                                              const csa_packed* packed, int32_t m, int32_t k, int32_t* idx,
                                              void* workspace, size_t workspace_bytes, void* stream) {
  using namespace csa;
  clear_error();
  CSA_REQUIRE(packed != nullptr, "csa_indexer_topk_packed: packed is NULL");
  CSA_REQUIRE(m >= 1, "csa_indexer_topk_packed: m must be >= 1");
  CSA_REQUIRE(k >= 1 && k <= kMaxK, "csa_indexer_topk_packed: k must be in [1, %d] (got %d)", kMaxK, k);
  CSA_REQUIRE(packed->n_seqs >= 0 && packed->max_tokens >= 0 && packed->total_tokens >= 0 &&
                  packed->total_tokens < (int64_t(1) << 31) && packed->total_entries >= 0 &&
                  packed->total_entries < (int64_t(1) << 31),
              "csa_indexer_topk_packed: bad packed descriptor sizes");
  if (packed->n_seqs == 0 || packed->total_tokens == 0) return CSA_OK;
  CSA_REQUIRE(packed->cu_tokens != nullptr && packed->cu_entries != nullptr,
              "csa_indexer_topk_packed: packed offsets are NULL");
  const int64_t max_n = (static_cast<int64_t>(packed->max_tokens) + m - 1) / m;
  if (max_n > kPrefillTcMaxN)
    return fail(CSA_ERR_UNSUPPORTED,
                "csa_indexer_topk_packed: sequences of up to %lld entries are supported (longest has %lld)",
                static_cast<long long>(kPrefillTcMaxN), static_cast<long long>(max_n));
  CSA_REQUIRE_PTR(qI);
  CSA_REQUIRE_PTR(wI);
  CSA_REQUIRE_PTR(kIc);
  CSA_REQUIRE_PTR(idx);
  const PackedLayout L = packed_layout(packed, m);
  if (workspace == nullptr || workspace_bytes < L.total)
    return fail(CSA_ERR_WORKSPACE, "csa_indexer_topk_packed: workspace of %zu bytes needed (got %zu)", L.total,
                workspace_bytes);
  CSA_REQUIRE(aligned16(workspace), "csa_indexer_topk_packed: workspace is not 16-byte aligned");
  int32_t* cu_grp = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + L.grp);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (csa_status st = check_launch("csa_indexer_topk_packed",
                                   launch_pdl(group_table_kernel, dim3(1), dim3(1024), 0, s, 1, packed->cu_tokens,
                                              static_cast<int>(packed->n_seqs), kPfQ, cu_grp));
      st != CSA_OK)
    return st;
  return launch_prefill_tc(qI, wI, kIc, 1, packed->total_tokens, 0, 0, m, k, idx, s, packed, cu_grp);
}
