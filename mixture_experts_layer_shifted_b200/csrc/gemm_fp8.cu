// Grouped GEMM on block-scaled FP8 operands (tcgen05.mma kind::mxf8f6f4 with
// E8M0 scales in tensor memory), for the FFN experts of an FP8 layer:
//   gate/up: H8[q, :] = quant(silu(X_e W_g,e^T) * (X_e W_u,e^T)), one [1,128] scale per 128 columns
//   down   : Y[q, :]  = H_e W_d,e^T, bf16
// q is a padded row: expert e's pairs occupy rows [128 mb_off[e], 128 mb_off[e] + count_e),
// so every row block of an expert starts on a 128-row boundary and its scales
// sit in whole scale atoms (layout in zc_fp8.cuh).
// (LongCat-Flash technical summary, zhangjingwei.cn, 六 推理與部署 定制內核:
// "量化" -- DeepSeek-V3's [1,128] activation / [128,128] weight blocks; the
// experts run as one grouped GEMM, "MoEGEMM".)
//
// The same kernel runs the W4A4 formats: MXFP4 (kind::mxf4, E8M0 scales per 32
// elements) and NVFP4 (kind::mxf4nvf4, UE4M3 scales per 16 elements, the
// weights' per-expert fp32 tensor scales applied to the accumulators), with
// 256-element k-blocks of packed E2M1 codes (four K=64 MMAs).
//
// Tile: 128 rows x 256 columns x 128-deep k-blocks (four K=32 MMAs); E4M3
// operands in 128-byte-swizzled K-major tiles; one fp32 accumulator of 256
// TMEM columns (the rest of TMEM holds the scales), drained by eight epilogue
// warps that release it as soon as their loads complete.  A scale atom covers
// four k-blocks, so the scales are copied into TMEM once every four k-blocks
// and each MMA picks its byte with the scale-factor id (k-block mod 4).
//
// Warp roles (320 threads): warp 0 loads (TMA tiles + bulk copies of scale
// atoms), warp 1 owns TMEM and issues the scale copies and MMAs (one thread),
// warps 2..9 drain TMEM: lane quarter = warp % 4, column half = (warp - 2) / 4.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zc_fp8.cuh"
#include "zc_internal.h"
#include "zc_ptx.cuh"

namespace zc {
namespace {

constexpr int BM = 128, BN = 256, BK = 128;
constexpr uint32_t A_BYTES = BM * BK;              // 16 KB
constexpr uint32_t B_BYTES = BN * BK;              // 32 KB
constexpr uint32_t TILE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 320;
constexpr int NUM_EPI = 256;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL = 256;                   // scale buffers: [256, 304) (FP8, MXFP4), [256, 352) (NVFP4)
constexpr uint32_t STG_BYTES = 32 * 64;           // down epilogue: a 32-row x 32-column bf16 box per warp

// Per mode and format: pipeline depth, scale bytes per stage (FP8 uses 3 atoms of its 6,
// MXFP4 6, NVFP4 12: one atom per operand 128 rows per K = 64 MMA) and the down epilogue's
// staging boxes (the gate/up epilogue stores from registers and has none).  The NVFP4 down
// GEMM keeps three stages: four would not fit beside the staging boxes.
template <int MODE, int FMT>
struct FmtCfg {
  static constexpr int kStages = (FMT == 2 && MODE == kDown) ? 3 : 4;
  static constexpr uint32_t kSfBytes = (FMT == 2 ? 12 : 6) * kAtomBytes;
  static constexpr uint32_t kStgBytes = MODE == kDown ? 8 * STG_BYTES : 0;
  static constexpr int kSmem = 1024 + kStages * (A_BYTES + B_BYTES + kSfBytes) + kStgBytes + 256 + 2 * 2 * BM * 4;
};
constexpr int cmax(int a, int b) { return a > b ? a : b; }
constexpr int SMEM_BYTES = cmax(cmax(FmtCfg<kGateUp, 0>::kSmem, FmtCfg<kDown, 0>::kSmem),
                                cmax(FmtCfg<kGateUp, 2>::kSmem, FmtCfg<kDown, 2>::kSmem));
static_assert(SMEM_BYTES <= 232448, "shared memory per block");

struct Tile {
  int64_t a_row;   // first padded A row (a multiple of 128)
  int rows_valid;  // rows of the tile that belong to the expert
  int b_row;       // first B row
  int n_blk;       // output column tile
  int grp;         // expert
};

__device__ __forceinline__ int total_tiles(const Fp8Args& a) { return a.mb_off[a.ngroups] * a.nblocks; }

template <int MODE>
__device__ __forceinline__ Tile decode_tile(const Fp8Args& a, int t) {
  int lo = 0, hi = a.ngroups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.mb_off[mid] * a.nblocks <= t) lo = mid;
    else hi = mid - 1;
  }
  const int g = lo;
  const int mb0 = a.mb_off[g];
  const int nmb = a.mb_off[g + 1] - mb0;
  const int local = t - mb0 * a.nblocks;
  Tile ti;
  ti.grp = g;
  ti.n_blk = local / nmb;
  const int m_blk = local - ti.n_blk * nmb;
  ti.a_row = (int64_t)(mb0 + m_blk) * BM;
  const int cnt = a.row_off[g + 1] - a.row_off[g];
  ti.rows_valid = min(BM, cnt - m_blk * BM);
  ti.b_row = g * a.b_rows_per_group + ti.n_blk * (MODE == kGateUp ? BN / 2 : BN);
  return ti;
}

// ------------------------------------------------------------------ block-scaled tcgen05
__device__ __forceinline__ void tc_cp_scales(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_mma_mxf8(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t tsfa,
                                            uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}
// Descriptor of a 512-byte scale atom read as 32 rows x 16 bytes, no swizzle
// (8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t atom_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(16u >> 4) << 16) | ((uint64_t)(128u >> 4) << 32) |
         ((uint64_t)1u << 46);
}
// Instruction descriptor, kind::mxf8f6f4 block-scaled: E4M3 A and B (K-major),
// fp32 D, E8M0 scales, scale-factor id `sf` for both operands.
__device__ __forceinline__ uint32_t idesc_mxf8(uint32_t sf) {
  return (sf << 4) | ((uint32_t)(BN >> 3) << 17) | (1u << 23) | ((uint32_t)(BM >> 4) << 24) | (sf << 29);
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_mma_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t tsfa,
                                            uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}
// kind::mxf4 block-scaled: E2M1 A and B (packed, K-major), fp32 D, E8M0 scales, K = 64;
// each MMA reads two scale bytes per row from byte `sf` (0 or 2).
__device__ __forceinline__ uint32_t idesc_mxf4(uint32_t sf) {
  return (sf << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | (1u << 23) | ((uint32_t)(BM >> 4) << 24) |
         (sf << 29);
}
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t tsfa,
                                            uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}
// kind::mxf4nvf4 with 16-element blocks: E2M1 A and B (packed, K-major), fp32 D, UE4M3
// scales (bit 23 clear), K = 64; each MMA reads four scale bytes per row (scale-factor id 0).
__device__ __forceinline__ uint32_t idesc_nvf4() {
  return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
// TMA store of one staged box at (x, y); completion tracked as a bulk group of this thread.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tm, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NUM_EPI) : "memory"); }

__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// All epilogue threads agree on `ok` (a barrier with an AND reduction), so they
// leave the tile loop together and never wait alone at the named barrier.
__device__ __forceinline__ bool epi_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)ok), "n"(NUM_EPI)
      : "memory");
  return r != 0;
}

// FMT 0: FP8 E4M3 with [1,128] / [128,128] scales (128 K per k-block, atoms loaded every
// fourth k-block); FMT 1: MXFP4 with [1,32] scales (256 K per k-block, six atoms every k-block);
// FMT 2: NVFP4 with [1,16] UE4M3 scales (256 K per k-block, twelve atoms every k-block) and the
// weights' per-expert fp32 scales applied to the accumulators in the epilogue.
template <int MODE, int FMT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_fp8_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
               const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmC,
               const Fp8Args args) {
  constexpr int STAGES = FmtCfg<MODE, FMT>::kStages;
  constexpr uint32_t SF_BYTES = FmtCfg<MODE, FMT>::kSfBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sSF = sB + STAGES * B_BYTES;
  uint8_t* sStg = sSF + STAGES * SF_BYTES;  // [epilogue warp] of STG_BYTES (down)
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + FmtCfg<MODE, FMT>::kStgBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 1;
  uint64_t* done = tempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  float* amax_s = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 256);  // [2][2][BM]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = args.err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, NUM_EPI);
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmA);
    tma_prefetch(&tmB0);
    if (MODE == kGateUp) tma_prefetch(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total = total_tiles(args);
  const int num_k = args.K / (FMT ? 2 * BK : BK);  // FP4 k-blocks hold 256 elements (128 bytes)

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- loads
      int stage = 0;
      uint32_t phase = 0;
      int fills = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile ti = decode_tile<MODE>(args, t);
        const int64_t atoms = (int64_t)args.groups_k * kAtomBytes;  // bytes of scale atoms per 128 rows
        const uint8_t* sfa = args.sfa + (ti.a_row >> 7) * atoms;
        const uint8_t* sfb_lo = args.sfb0 + (int64_t)(ti.b_row >> 7) * atoms;
        const uint8_t* sfb_hi = (MODE == kGateUp) ? args.sfb1 + (int64_t)(ti.b_row >> 7) * atoms : sfb_lo + atoms;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, err, 11)) {
            ok = false;
            break;
          }
          const bool with_sf = FMT ? true : (kb & 3) == 0;
          uint8_t* a_dst = sA + stage * A_BYTES;
          uint8_t* b_dst = sB + stage * B_BYTES;
          mbar_expect_tx(&full[stage], TILE_BYTES + (with_sf ? (FMT == 2 ? 12u : FMT ? 6u : 3u) * kAtomBytes : 0u));
          tma_load_2d(a_dst, &tmA, kb * BK, (int)ti.a_row, &full[stage]);
          if (MODE == kGateUp) {
            tma_load_2d(b_dst, &tmB0, kb * BK, ti.b_row, &full[stage]);
            tma_load_2d(b_dst + B_BYTES / 2, &tmB1, kb * BK, ti.b_row, &full[stage]);
          } else {
            tma_load_2d(b_dst, &tmB0, kb * BK, ti.b_row, &full[stage]);
          }
          uint8_t* sf_dst = sSF + stage * SF_BYTES;
          if (FMT == 0 && with_sf) {
            const int64_t g = (int64_t)(kb >> 2) * kAtomBytes;
            bulk_load(sf_dst, sfa + g, kAtomBytes, &full[stage]);
            bulk_load(sf_dst + kAtomBytes, sfb_lo + g, kAtomBytes, &full[stage]);
            bulk_load(sf_dst + 2 * kAtomBytes, sfb_hi + g, kAtomBytes, &full[stage]);
          } else if (FMT == 1) {
            // K groups 2kb, 2kb+1: [A g0][A g1][B lo g0][B hi g0][B lo g1][B hi g1]
            const int64_t g = (int64_t)(2 * kb) * kAtomBytes;
            bulk_load(sf_dst, sfa + g, kAtomBytes, &full[stage]);
            bulk_load(sf_dst + kAtomBytes, sfa + g + kAtomBytes, kAtomBytes, &full[stage]);
            bulk_load(sf_dst + 2 * kAtomBytes, sfb_lo + g, kAtomBytes, &full[stage]);
            bulk_load(sf_dst + 3 * kAtomBytes, sfb_hi + g, kAtomBytes, &full[stage]);
            bulk_load(sf_dst + 4 * kAtomBytes, sfb_lo + g + kAtomBytes, kAtomBytes, &full[stage]);
            bulk_load(sf_dst + 5 * kAtomBytes, sfb_hi + g + kAtomBytes, kAtomBytes, &full[stage]);
          } else if (FMT == 2) {
            // K groups 4kb .. 4kb+3 (one per MMA), consecutive in memory: [A][B lo][B hi] x 4 atoms
            const int64_t g = (int64_t)(4 * kb) * kAtomBytes;
            bulk_load(sf_dst, sfa + g, 4 * kAtomBytes, &full[stage]);
            bulk_load(sf_dst + 4 * kAtomBytes, sfb_lo + g, 4 * kAtomBytes, &full[stage]);
            bulk_load(sf_dst + 8 * kAtomBytes, sfb_hi + g, 4 * kAtomBytes, &full[stage]);
          }
          ++fills;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // no copy may still be in flight when the CTA exits
      const int pending = fills < STAGES ? fills : STAGES;
      for (int i = 0; i < pending; ++i) {
        if (--stage < 0) {
          stage = STAGES - 1;
          phase ^= 1u;
        }
        mbar_wait(&full[stage], phase, err, 19);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- scale copies + MMAs
      // descriptors of stage 0; a stage's tiles start A_BYTES / B_BYTES further on, and
      // the start-address field counts 16-byte units
      const uint64_t adesc0 = sw128_kmajor_desc(smem_u32(sA)), bdesc0 = sw128_kmajor_desc(smem_u32(sB));
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!mbar_wait(tempty, acc_phase ^ 1u, err, 12)) break;
        tc_fence_after();
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&full[stage], phase, err, 13)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sd = smem_u32(sSF + stage * SF_BYTES);
          if (FMT == 0) {
            const uint32_t sfa_t = tmem_base + SF_COL + 16u * (uint32_t)((kb >> 2) & 1);
            const uint32_t sfb_t = sfa_t + 4;
            if ((kb & 3) == 0) {
              tc_cp_scales(sfa_t, atom_desc(sd));
              tc_cp_scales(sfb_t, atom_desc(sd + kAtomBytes));
              tc_cp_scales(sfb_t + 4, atom_desc(sd + 2 * kAtomBytes));
            }
            const uint32_t sf = (uint32_t)(kb & 3);
            const uint32_t idesc = idesc_mxf8(sf);
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
              tc_mma_mxf8(tmem_base, adesc0 + (uint64_t)(stage * (A_BYTES >> 4) + kk * 2),
                          bdesc0 + (uint64_t)(stage * (B_BYTES >> 4) + kk * 2), idesc, (sf << 30) | sfa_t,
                          (sf << 30) | sfb_t, (kb | kk) != 0 ? 1u : 0u);
          } else if (FMT == 1) {
            // TMEM scales of this k-block: A g0 +0, A g1 +4, B g0 +8 (rows 0..127) / +12 (128..255), B g1 +16 / +20
            const uint32_t buf = tmem_base + SF_COL + 24u * (uint32_t)(kb & 1);
#pragma unroll
            for (int a = 0; a < 6; ++a) tc_cp_scales(buf + 4 * a, atom_desc(sd + a * kAtomBytes));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {  // K = 64 each: 32 bytes of the 128-byte rows
              const uint32_t sf = (uint32_t)((kk & 1) * 2);
              const uint32_t g = (uint32_t)(kk >> 1);
              tc_mma_mxf4(tmem_base, adesc0 + (uint64_t)(stage * (A_BYTES >> 4) + kk * 2),
                          bdesc0 + (uint64_t)(stage * (B_BYTES >> 4) + kk * 2), idesc_mxf4(sf),
                          (sf << 30) | (buf + 4 * g), (sf << 30) | (buf + 8 + 8 * g), (kb | kk) != 0 ? 1u : 0u);
            }
          } else {
            // TMEM scales of this k-block, one 4-column group per atom: A for MMA kk at +4kk, B at
            // +16+8kk (rows 0..127) and +20+8kk (rows 128..255)
            const uint32_t buf = tmem_base + SF_COL + 48u * (uint32_t)(kb & 1);
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              tc_cp_scales(buf + 4 * a, atom_desc(sd + a * kAtomBytes));
              tc_cp_scales(buf + 16 + 8 * a, atom_desc(sd + (4 + a) * kAtomBytes));
              tc_cp_scales(buf + 20 + 8 * a, atom_desc(sd + (8 + a) * kAtomBytes));
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // K = 64 each: 32 bytes of the 128-byte rows
              tc_mma_nvf4(tmem_base, adesc0 + (uint64_t)(stage * (A_BYTES >> 4) + kk * 2),
                          bdesc0 + (uint64_t)(stage * (B_BYTES >> 4) + kk * 2), idesc_nvf4(), buf + 4 * kk,
                          buf + 16 + 8 * kk, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull);
        acc_phase ^= 1u;
      }
      // every MMA and copy of this CTA has completed before TMEM is released
      tc_commit(done);
      mbar_wait(done, 0, err, 14);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2..9)
    const int quarter = warp & 3;           // TMEM lanes [32*quarter, 32*quarter + 32)
    const int half = (warp - 2) >> 2;       // column half of the tile
    const int row = quarter * 32 + lane;
    const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16);
    uint32_t acc_phase = 0;
    int buf = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile ti = decode_tile<MODE>(args, t);
      // NVFP4: the weights' tensor scales (gate/up: W_g's and W_u's; down: W_d's)
      float s0 = 1.0f, s1 = 1.0f;
      if (FMT == 2) {
        s0 = __ldg(args.gsc0 + ti.grp);
        if (MODE == kGateUp) s1 = __ldg(args.gsc1 + ti.grp);
      }
      const bool got = mbar_wait(tfull, acc_phase, err, 15);
      if (MODE == kGateUp && FMT == 0) {
        if (!epi_all(got)) break;
      } else if (!got) {
        break;
      }
      tc_fence_after();
      const bool row_ok = row < ti.rows_valid;
      const int64_t grow = ti.a_row + row;
      if (MODE == kGateUp) {
        // gate columns [64 half, +64) and the matching up columns [128 + 64 half, +64)
        uint32_t g0[32], g1[32], u0[32], u1[32];
        tmem_ld32(tbase + 64 * half, g0);
        tmem_ld32(tbase + 64 * half + 32, g1);
        tmem_ld32(tbase + BN / 2 + 64 * half, u0);
        tmem_ld32(tbase + BN / 2 + 64 * half + 32, u1);
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(tempty);  // the accumulator may be overwritten from here on
        float amax = 0.0f, am0 = 0.0f, am1 = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float h0 = FMT == 2 ? silu_mul(__uint_as_float(g0[j]) * s0, __uint_as_float(u0[j]) * s1)
                                    : silu_mul(__uint_as_float(g0[j]), __uint_as_float(u0[j]));
          const float h1 = FMT == 2 ? silu_mul(__uint_as_float(g1[j]) * s0, __uint_as_float(u1[j]) * s1)
                                    : silu_mul(__uint_as_float(g1[j]), __uint_as_float(u1[j]));
          g0[j] = __float_as_uint(h0);
          g1[j] = __float_as_uint(h1);
          am0 = fmaxf(am0, fabsf(h0));
          am1 = fmaxf(am1, fabsf(h1));
        }
        amax = fmaxf(am0, am1);
        if (FMT == 1) {
          // [1,32] blocks: columns [64 half, +32) and [64 half + 32, +32) of this H block
          const int col0 = ti.n_blk * (BN / 2) + 64 * half;
          if (row_ok && col0 < args.n_out) {
            uint8_t* dst = static_cast<uint8_t*>(args.out) + grow * args.ldo + (col0 >> 1);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const uint32_t* h = q == 0 ? g0 : g1;
              const uint32_t code = mx4_code(q == 0 ? am0 : am1);
              const float inv = e8m0_inverse(code);
              float f[8];
              uint4 v;
              uint32_t* vw = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
              for (int w = 0; w < 4; ++w) {
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(h[8 * w + i]);
                vw[w] = pack_e2m1x8(f, inv);
              }
              *reinterpret_cast<uint4*>(dst + 16 * q) = v;
              args.out_sf[atom_offset(grow, (col0 >> 5) + q, args.out_groups)] = (uint8_t)code;
            }
          }
          acc_phase ^= 1u;
          buf ^= 1;
          continue;
        }
        if (FMT == 2) {
          // [1,16] blocks (g = 1): columns [64 half + 16 q, +16) of this H block, q = 0..3
          const int col0 = ti.n_blk * (BN / 2) + 64 * half;
          if (row_ok && col0 < args.n_out) {
            uint8_t* dst = static_cast<uint8_t*>(args.out) + grow * args.ldo + (col0 >> 1);
            uint32_t w[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t* h = (q < 2 ? g0 : g1) + 16 * (q & 1);
              float f[16];
              float am = 0.0f;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                f[i] = __uint_as_float(h[i]);
                am = fmaxf(am, fabsf(f[i]));
              }
              const uint32_t code = nv4_code(am, 1.0f);
              const float inv = nv4_inverse(code, 1.0f);
              w[2 * q] = pack_e2m1x8(f, inv);
              w[2 * q + 1] = pack_e2m1x8(f + 8, inv);
              args.out_sf[atom_offset(grow, (col0 >> 4) + q, args.out_groups)] = (uint8_t)code;
            }
            *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(dst + 16) = make_uint4(w[4], w[5], w[6], w[7]);
          }
          acc_phase ^= 1u;
          buf ^= 1;
          continue;
        }
        // the row's [1,128] block spans both halves: exchange the partial maxima
        amax_s[(buf * 2 + half) * BM + row] = amax;
        epi_sync();
        amax = fmaxf(amax, amax_s[(buf * 2 + (half ^ 1)) * BM + row]);
        const uint32_t code = e8m0_code(amax);
        const float inv = e8m0_inverse(code);
        const int col0 = ti.n_blk * (BN / 2) + 64 * half;
        if (row_ok && col0 < args.n_out) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out) + grow * args.ldo + col0);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const uint32_t* h = q == 0 ? g0 : g1;
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              uint4 v;
              v.x = pack_e4m3x4(__uint_as_float(h[16 * w + 0]) * inv, __uint_as_float(h[16 * w + 1]) * inv,
                                __uint_as_float(h[16 * w + 2]) * inv, __uint_as_float(h[16 * w + 3]) * inv);
              v.y = pack_e4m3x4(__uint_as_float(h[16 * w + 4]) * inv, __uint_as_float(h[16 * w + 5]) * inv,
                                __uint_as_float(h[16 * w + 6]) * inv, __uint_as_float(h[16 * w + 7]) * inv);
              v.z = pack_e4m3x4(__uint_as_float(h[16 * w + 8]) * inv, __uint_as_float(h[16 * w + 9]) * inv,
                                __uint_as_float(h[16 * w + 10]) * inv, __uint_as_float(h[16 * w + 11]) * inv);
              v.w = pack_e4m3x4(__uint_as_float(h[16 * w + 12]) * inv, __uint_as_float(h[16 * w + 13]) * inv,
                                __uint_as_float(h[16 * w + 14]) * inv, __uint_as_float(h[16 * w + 15]) * inv);
              dst[q * 2 + w] = v;
            }
          }
          if (half == 0) args.out_sf[atom_offset(grow, ti.n_blk, args.out_groups)] = (uint8_t)code;
        }
      } else {
        uint32_t r[4][32];
#pragma unroll
        for (int i = 0; i < 4; ++i) tmem_ld32(tbase + 128 * half + 32 * i, r[i]);
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(tempty);
        // NVFP4: W_d's tensor scale on the way out
        auto f = [s0](uint32_t b) { return FMT == 2 ? __uint_as_float(b) * s0 : __uint_as_float(b); };
        // a row group whose 32 rows are all valid leaves by TMA stores of 32 x 32 boxes staged
        // in shared memory; a partly valid group (an expert's last rows: few at decode) by row
        // stores of its valid rows
        const int col0 = ti.n_blk * BN + 128 * half;
        if (col0 < args.n_out && quarter * 32 + 32 > ti.rows_valid) {
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out) + grow * args.ldo + col0);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int q = 0; q < 4; ++q)
                dst[i * 4 + q] =
                    make_uint4(pack_bf16(f(r[i][8 * q + 0]), f(r[i][8 * q + 1])),
                               pack_bf16(f(r[i][8 * q + 2]), f(r[i][8 * q + 3])),
                               pack_bf16(f(r[i][8 * q + 4]), f(r[i][8 * q + 5])),
                               pack_bf16(f(r[i][8 * q + 6]), f(r[i][8 * q + 7])));
          }
        } else if (col0 < args.n_out) {  // the same for the whole warp
          uint8_t* stg = sStg + (warp - 2) * STG_BYTES;
          const int grow0 = (int)ti.a_row + quarter * 32;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (lane == 0) bulk_wait_read_0();  // the previous box has been read out
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q)
              *reinterpret_cast<uint4*>(stg + lane * 64 + q * 16) =
                  make_uint4(pack_bf16(f(r[i][8 * q + 0]), f(r[i][8 * q + 1])),
                             pack_bf16(f(r[i][8 * q + 2]), f(r[i][8 * q + 3])),
                             pack_bf16(f(r[i][8 * q + 4]), f(r[i][8 * q + 5])),
                             pack_bf16(f(r[i][8 * q + 6]), f(r[i][8 * q + 7])));
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmC, stg, col0 + 32 * i, grow0);
              bulk_commit();
            }
          }
        }
      }
      acc_phase ^= 1u;
      buf ^= 1;
    }
    if (MODE == kDown && lane == 0) bulk_wait_all();  // every store complete before exit
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int MODE, int FMT>
cudaError_t launch_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const CUtensorMap& c,
                        const Fp8Args& args, int grid, cudaStream_t s) {
  static SmemAttr attr{};
  constexpr int smem = FmtCfg<MODE, FMT>::kSmem;
  const cudaError_t e = ensure_smem_attr(attr, k_fp8_gemm<MODE, FMT>, smem);
  if (e != cudaSuccess) return e;
  k_fp8_gemm<MODE, FMT><<<grid, NUM_THREADS, smem, s>>>(a, b0, b1, c, args);
  return cudaGetLastError();
}

}  // namespace

int fp8_smem_bytes() { return SMEM_BYTES; }
int fp8_block_n(int mode) { return mode == kGateUp ? BN / 2 : BN; }

cudaError_t launch_fp8_gemm(int mode, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                            const CUtensorMap& c, const Fp8Args& args, int grid, cudaStream_t s) {
  if (args.fmt < 0 || args.fmt > 2 || (args.fmt == 2 && (!args.gsc0 || (mode == kGateUp && !args.gsc1))))
    return cudaErrorInvalidValue;
  if (mode == kGateUp) {
    if (args.fmt == 2) return launch_mode<kGateUp, 2>(a, b0, b1, c, args, grid, s);
    return args.fmt ? launch_mode<kGateUp, 1>(a, b0, b1, c, args, grid, s)
                    : launch_mode<kGateUp, 0>(a, b0, b1, c, args, grid, s);
  }
  if (mode == kDown) {
    if (args.fmt == 2) return launch_mode<kDown, 2>(a, b0, b1, c, args, grid, s);
    return args.fmt ? launch_mode<kDown, 1>(a, b0, b1, c, args, grid, s)
                    : launch_mode<kDown, 0>(a, b0, b1, c, args, grid, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace zc
