// Grouped output projection after the core attention.
//
// DeepSeek-V4 paper summary (hyper.ai), section "Method", CSA paragraph: the
// MQA core attention is followed by a grouped output projection that keeps its
// compute cost down.  The H heads form G groups of H/G consecutive heads; the
// outputs of group g, concatenated head after head (K = (H/G) * 128 values per
// query row), are multiplied by the group's own weight W[g] (d_g x K):
//     y[r, g, :] = x_g[r, :] . W[g]^T,   x_g[r] = o[r, g*H/G .. (g+1)*H/G - 1, :]
// i.e. G independent GEMMs [R x K] x [K x d_g] (a block-diagonal projection).
//
// One persistent tcgen05 kernel runs all of them.  Output tiles are 128 rows x
// BN channels of one group, taken in the order (row tile, group, channel tile)
// so that the CTAs working at the same time share their A rows in L2.  Warp 0
// streams 64-wide K slices of A (attention outputs) and B (weights) by TMA
// (128-byte swizzle, no multicast) into a ring of shared-memory stages; one
// thread of warp 1 issues the MMAs (M = 128, N = BN, bf16 in, fp32 in TMEM);
// warps 2-5 drain the accumulator (thread = row) to bf16 while the next tile
// accumulates into the other TMEM buffer.  All mbarrier waits are bounded.
//
// The projection is not fused into the attention kernels: those own one query
// row per CTA, while the projection needs 128-row tiles to reuse each weight
// slice across rows (the weights of one group are d_g x K bf16, 2 MiB at
// d_g = K = 1024).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "host_util.h"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int kOpM = 128;        // rows per tile (TMEM lanes)
constexpr int kOpK = 64;         // K per stage: one 128-byte swizzle atom of bf16
constexpr int kOpThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

template <int BN>
struct OpShape {
  static constexpr int kABytes = kOpM * kOpK * 2;
  static constexpr int kBBytes = BN * kOpK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = BN >= 256 ? 4 : (BN >= 128 ? 5 : 6);
  static constexpr size_t kBarOff = static_cast<size_t>(kStages) * kStageBytes;
  static constexpr size_t kSmem = kBarOff + 256 + 1024;  // barriers + alignment slack
  static constexpr uint32_t kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;
};

struct OpParams {
  int64_t R;
  int G, K, dg;
  int m_tiles, n_tiles;
  __nv_bfloat16* y;  // [R, G, dg]
};

template <int BN>
__global__ void __launch_bounds__(kOpThreads, 1) out_proj_kernel(OpParams p, const __grid_constant__ CUtensorMap amap,
                                                                 const __grid_constant__ CUtensorMap bmap) {
  pdl_wait();
  using S = OpShape<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);  // [kStages] stage loaded
  uint64_t* empty = full + S::kStages;                               // [kStages] stage consumed by the MMAs
  uint64_t* tfull = empty + S::kStages;                              // [2] accumulator complete
  uint64_t* tempty = tfull + 2;                                      // [2] accumulator drained
  uint32_t* tslot = reinterpret_cast<uint32_t*>(tempty + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kc_n = p.K / kOpK;
  const int64_t tiles = static_cast<int64_t>(p.m_tiles) * p.G * p.n_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S::kStages; ++i) {
      tc::bar_init(&full[i], 1);
      tc::bar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::bar_init(&tfull[i], 1);
      tc::bar_init(&tempty[i], 4 * 32);
    }
    tc::bar_init_fence();
  }
  if (warp == 1) tc::tmem_alloc(tslot, S::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    // ===================== TMA producer =====================
    if (lane == 0) {
      bool healthy = true;
      int64_t it = 0;
      for (int64_t tile = blockIdx.x; tile < tiles && healthy; tile += gridDim.x) {
        const int n = static_cast<int>(tile % p.n_tiles);
        const int64_t mg = tile / p.n_tiles;
        const int g = static_cast<int>(mg % p.G);
        const int m = static_cast<int>(mg / p.G);
        for (int kc = 0; kc < kc_n; ++kc, ++it) {
          const int st = static_cast<int>(it % S::kStages);
          if (it >= S::kStages && !tc::bar_wait(&empty[st], static_cast<uint32_t>(((it / S::kStages) - 1) & 1))) {
            healthy = false;
            break;
          }
          uint8_t* a = smem + st * S::kStageBytes;
          tc::bar_arrive_expect_tx(&full[st], S::kStageBytes);
          tc::tma_load_2d(a, &amap, g * p.K + kc * kOpK, m * kOpM, &full[st]);
          tc::tma_load_2d(a + S::kABytes, &bmap, kc * kOpK, g * p.dg + n * BN, &full[st]);
        }
      }
    }
  } else if (warp == 1) {
    // ===================== MMA issue (one thread) =====================
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16(kOpM, BN, false, false);
      bool healthy = true;
      int64_t it = 0;
      int tcount = 0;
      for (int64_t tile = blockIdx.x; tile < tiles && healthy; tile += gridDim.x, ++tcount) {
        const int acc = tcount & 1;
        if (tcount >= 2 && !tc::bar_wait(&tempty[acc], static_cast<uint32_t>(((tcount >> 1) - 1) & 1))) break;
        tc::fence_after_sync();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * BN);
        for (int kc = 0; kc < kc_n; ++kc, ++it) {
          const int st = static_cast<int>(it % S::kStages);
          if (!tc::bar_wait(&full[st], static_cast<uint32_t>((it / S::kStages) & 1))) {
            healthy = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t a = smem_u32(smem + st * S::kStageBytes);
          const uint32_t b = a + S::kABytes;
#pragma unroll
          for (int k4 = 0; k4 < kOpK / 16; ++k4)
            tc::mma_bf16_ss(d, tc::desc_sw128(a + k4 * 32, 16, 1024), tc::desc_sw128(b + k4 * 32, 16, 1024), idesc,
                            (kc | k4) != 0 ? 1u : 0u);
          tc::mma_commit(&empty[st]);
        }
        tc::mma_commit(&tfull[acc]);
      }
    }
  } else {
    // ===================== epilogue: thread = accumulator row =====================
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int tcount = 0;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tcount) {
      const int n = static_cast<int>(tile % p.n_tiles);
      const int64_t mg = tile / p.n_tiles;
      const int g = static_cast<int>(mg % p.G);
      const int64_t m = mg / p.G;
      const int acc = tcount & 1;
      if (!tc::bar_wait(&tfull[acc], static_cast<uint32_t>((tcount >> 1) & 1))) break;
      tc::fence_after_sync();
      const int64_t row = m * kOpM + q * 32 + lane;
      __nv_bfloat16* dst = p.y + (row * p.G + g) * p.dg + static_cast<int64_t>(n) * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tc::tmem_ld32(tmem + lane_base + static_cast<uint32_t>(acc * BN + c * 32), v);
        if (row < p.R) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            reinterpret_cast<uint4*>(dst + c * 32)[j] =
                make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                           pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
        }
      }
      tc::fence_before_sync();
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(&tempty[acc])) : "memory");
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, S::kTmemCols);
}

csa_status encode_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                     uint32_t box_cols, uint32_t box_rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return fail(CSA_ERR_CUDA, "csa_grouped_out_proj: cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA_ERR_CUDA, "csa_grouped_out_proj: tensor map encoding failed (%d)", int(r));
  return CSA_OK;
}

template <int BN>
csa_status launch_out_proj(const OpParams& p, const CUtensorMap& amap, const CUtensorMap& bmap, cudaStream_t s) {
  using S = OpShape<BN>;
  if (!ensure_smem(reinterpret_cast<const void*>(out_proj_kernel<BN>), static_cast<int>(S::kSmem)))
    return fail(CSA_ERR_CUDA, "csa_grouped_out_proj: cannot raise the shared memory limit");
  const int64_t tiles = static_cast<int64_t>(p.m_tiles) * p.G * p.n_tiles;
  const int grid = static_cast<int>(tiles < num_sms() ? tiles : num_sms());
  prof_begin(s);
  const cudaError_t e = launch_pdl(out_proj_kernel<BN>, dim3(grid), dim3(kOpThreads), S::kSmem, s, 1, p, amap, bmap);
  prof_end(s);
  return check_launch("csa_grouped_out_proj", e);
}

}  // namespace
}  // namespace csa

extern "C" csa_status csa_grouped_out_proj(const void* o, int64_t R, int32_t H, int32_t G, int32_t d_g,
                                           const void* w, void* y, void* stream) {
  using namespace csa;
  clear_error();
  CSA_REQUIRE(R >= 0 && R < (int64_t(1) << 31), "csa_grouped_out_proj: R must be in [0, 2^31)");
  CSA_REQUIRE(H >= 1 && H <= 256 && G >= 1 && H % G == 0, "csa_grouped_out_proj: G must divide H (H %d, G %d)", H, G);
  CSA_REQUIRE(d_g >= 64 && d_g % 64 == 0 && d_g <= 65536, "csa_grouped_out_proj: d_g must be a multiple of 64 (got %d)",
              d_g);
  if (R == 0) return CSA_OK;
  CSA_REQUIRE_PTR(o);
  CSA_REQUIRE_PTR(w);
  CSA_REQUIRE_PTR(y);
  OpParams p;
  p.R = R;
  p.G = G;
  p.K = (H / G) * kDV;
  p.dg = d_g;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.m_tiles = static_cast<int>((R + kOpM - 1) / kOpM);
  // wide tiles when there are rows enough to fill the device, narrow ones otherwise
  const int64_t wide_tiles = static_cast<int64_t>(p.m_tiles) * G * (d_g / 256);
  const int bn = (d_g % 256 == 0 && wide_tiles >= num_sms()) ? 256 : (d_g % 128 == 0 && R > kOpM ? 128 : 64);
  p.n_tiles = d_g / bn;
  CUtensorMap amap, bmap;
  memset(&amap, 0, sizeof(amap));
  memset(&bmap, 0, sizeof(bmap));
  const uint64_t hk = static_cast<uint64_t>(H) * kDV;
  if (csa_status st = encode_2d(&amap, o, hk, static_cast<uint64_t>(R), hk * 2, kOpK, kOpM); st != CSA_OK) return st;
  if (csa_status st = encode_2d(&bmap, w, static_cast<uint64_t>(p.K), static_cast<uint64_t>(G) * d_g,
                                static_cast<uint64_t>(p.K) * 2, kOpK, static_cast<uint32_t>(bn));
      st != CSA_OK)
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (bn == 256) return launch_out_proj<256>(p, amap, bmap, s);
  if (bn == 128) return launch_out_proj<128>(p, amap, bmap, s);
  return launch_out_proj<64>(p, amap, bmap, s);
}

namespace csa {
// Reads (and optionally clears) this unit's device error word.
CSA_DEFINE_DEVICE_ERROR_READER(out_proj_device_error)
}  // namespace csa

