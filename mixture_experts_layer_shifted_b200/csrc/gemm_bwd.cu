// Tensor-core GEMMs of the backward pass (bf16 operands, fp32 accumulation in TMEM).
//
// LongCat-Flash technical summary (zhangjingwei.cn), 五 訓練基礎設施: the MoE layer
// trains with a fused GemmAdd (the fp32 gradient addition done in the GEMM's
// epilogue, so the product is never written out and re-read) and a
// deterministic ScatterAdd.  One persistent, warp-specialised kernel template
// (the forward's structure: warp 0 loads, warp 1 issues tcgen05.mma, warps 2..5
// drain TMEM, two 256-column accumulators) serves every contraction:
//
//   SCHED_ROWS  (rows of an expert's tokens x output columns, K fixed):
//     dH  = dY W_d                 A dY (K-major)      B W_d (MN-major)          -> bf16, or (the forward
//                                  saved G and U) the SwiGLU backward in the epilogue -> dG, dU, H
//     [G|U] = X [W_g; W_u]^T       A X  (K-major)      B W_g / W_u (K-major)     -> SwiGLU backward epilogue
//     dX  = [dG|dU] [W_g; W_u]     A dGU (K-major)     B W_g then W_u (MN-major) -> bf16
//     dx_router = dl W_r           A dl (K-major)      B W_r (MN-major)          -> bf16
//   SCHED_WGRAD (output rows x output columns of one expert, K = its tokens):
//     dW_d += dY_e^T H_e,  dW_g += dG_e^T X_e,  dW_u += dU_e^T X_e,  dW_r += dl^T x
//                                  A, B both MN-major (token-major activations) -> fp32 GemmAdd
//
// Token rows are padded: expert e's pairs occupy rows [128 mb_off[e], 128 mb_off[e] + count_e)
// of every row-indexed buffer, and the padding rows hold zeros, so a weight
// gradient's reduction over an expert's rows can run over whole 64-row k-blocks.
//
// Operand tiles in shared memory, 128-byte swizzle: K-major = rows of 64 K
// elements (128 B); MN-major = boxes of 64 M (or N) elements x 64 K rows, box i
// 8 KB after box i-1; the MMA descriptor's leading offset is then 8 KB (next box)
// and its stride offset 1 KB (next 8 K rows), and a K=16 step advances 2 KB.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zc_internal.h"
#include "zc_ptx.cuh"

namespace zc {
namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr uint32_t A_BYTES = BM * BK * 2;
constexpr uint32_t B_BYTES = BN * BK * 2;
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr uint32_t STG_BYTES = 32 * 32 * 4;  // GemmAdd staging: 32 rows x 32 fp32 per warp and buffer

// Operand stages, and GemmAdd staging buffers per epilogue warp (reduce-adds in flight).
constexpr int kRowStages = 4;
constexpr int kWgStages = 4, kWgBufs = 2;
template <int EPI>
struct Cfg {
  static constexpr int kStages = EPI == kEpiAddF32 ? kWgStages : kRowStages;
  // staging buffers per epilogue warp: GemmAdd boxes, or the bf16 outputs' TMA-store boxes
  //   (the saved-SwiGLU epilogue uses its warp's two buffers as dG, dU, H boxes of 2 KB each)
  static constexpr int kBufs = EPI == kEpiAddF32 ? kWgBufs : (EPI == kEpiBf16 || EPI == kEpiSwigluSaved ? 2 : 0);
  static constexpr int kSmem = 1024 + kStages * STAGE_BYTES + 4 * kBufs * STG_BYTES + 256;
  static_assert(kSmem <= 232448, "shared memory per block");
};

struct Tile {
  int64_t a_row;   // SCHED_ROWS: first padded A row; SCHED_WGRAD: first K row (padded token row)
  int rows_valid;  // SCHED_ROWS: rows of the tile that belong to the expert
  int num_k;       // k-blocks of this tile (0: nothing to do)
  int g;           // expert
  int m_blk, n_blk;
};

template <int SCHED>
__device__ __forceinline__ int total_tiles(const BwdArgs& a) {
  if (SCHED == kSchedRows) return a.mb_off[a.ngroups] * a.nblocks;
  return a.ngroups * a.mblocks * a.nblocks;
}

template <int SCHED>
__device__ __forceinline__ Tile decode_tile(const BwdArgs& a, int t) {
  Tile ti;
  if (SCHED == kSchedRows) {
    // expert-major, then column tile, then row block (as the forward)
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
    ti.g = g;
    ti.n_blk = local / nmb;
    ti.m_blk = local - ti.n_blk * nmb;
    ti.a_row = (int64_t)(mb0 + ti.m_blk) * BM;
    ti.rows_valid = min(BM, a.row_off[g + 1] - a.row_off[g] - ti.m_blk * BM);
    ti.num_k = a.K / BK;
  } else {
    const int per_g = a.mblocks * a.nblocks;
    ti.g = t / per_g;
    const int local = t - ti.g * per_g;
    ti.n_blk = local / a.mblocks;
    ti.m_blk = local - ti.n_blk * a.mblocks;
    ti.a_row = (int64_t)a.mb_off[ti.g] * BM;
    ti.rows_valid = BM;
    ti.num_k = (a.mb_off[ti.g + 1] - a.mb_off[ti.g]) * (BM / BK);
  }
  return ti;
}

// 128-byte-swizzled MN-major descriptor: boxes of 64 MN elements 8 KB apart
// (leading offset), 8-row K groups 1 KB apart (stride offset).
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(8192u >> 4) << 16) | ((uint64_t)(1024u >> 4) << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// TMA reduce-add of a 32 x 32 fp32 box (128-byte swizzled in shared memory) into
// the accumulator at (n, m, g); completion tracked as a bulk group of this thread.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* tm, const void* src, int n, int m, int g) {
  asm volatile("cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(smem_u32(src)), "r"(n), "r"(m), "r"(g)
               : "memory");
}
// TMA store of a 32-row x 64-column bf16 box (128-byte swizzled in shared memory) at (x, y).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tm, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
// TMA store of a 32 x 32 fp32 box (the same staging and tensor map): the overwrite mode.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* tm, const void* src, int n, int m, int g) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(smem_u32(src)), "r"(n), "r"(m), "r"(g)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

template <int SCHED, bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_bwd_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
               const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmC,
               const BwdArgs args) {
  constexpr int STAGES = Cfg<EPI>::kStages, NBUF = Cfg<EPI>::kBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sStg = sB + STAGES * B_BYTES;  // 1024-aligned: [warp quarter][buffer] of STG_BYTES
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + 4 * NBUF * STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = args.err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmA);
    tma_prefetch(&tmB0);
    tma_prefetch(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = total_tiles<SCHED>(args);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int fills = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile ti = decode_tile<SCHED>(args, t);
        for (int kb = 0; kb < ti.num_k; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, err, 21)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = sA + stage * A_BYTES;
          uint8_t* b_dst = sB + stage * B_BYTES;
          mbar_expect_tx(&full[stage], STAGE_BYTES);
          if (SCHED == kSchedRows) {
            tma_load_2d(a_dst, &tmA, args.a_col0 + kb * BK, (int)ti.a_row, &full[stage]);  // K-major A
            if (!B_MN) {
              // W_g rows then the same W_u rows (SwiGLU pairs in one tile)
              const int brow = (int)(ti.g * args.b_row_per_group) + ti.n_blk * (BN / 2);
              tma_load_2d(b_dst, &tmB0, kb * BK, brow, &full[stage]);
              tma_load_2d(b_dst + B_BYTES / 2, &tmB1, kb * BK, brow, &full[stage]);
            } else {
              const bool second = kb * BK >= args.k_split;
              const int krow = (int)(ti.g * args.b_row_per_group) + kb * BK - (second ? args.k_split : 0);
#pragma unroll
              for (int i = 0; i < BN / 64; ++i)
                tma_load_2d(b_dst + i * 8192, second ? &tmB1 : &tmB0, ti.n_blk * BN + 64 * i, krow, &full[stage]);
            }
          } else {
            const int krow = (int)ti.a_row + kb * BK;
#pragma unroll
            for (int i = 0; i < BM / 64; ++i)
              tma_load_2d(a_dst + i * 8192, &tmA, args.a_col0 + ti.m_blk * BM + 64 * i, krow, &full[stage]);
#pragma unroll
            for (int i = 0; i < BN / 64; ++i)
              tma_load_2d(b_dst + i * 8192, &tmB0, ti.n_blk * BN + 64 * i, krow, &full[stage]);
          }
          ++fills;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      const int pending = fills < STAGES ? fills : STAGES;
      for (int i = 0; i < pending; ++i) {
        if (--stage < 0) {
          stage = STAGES - 1;
          phase ^= 1u;
        }
        mbar_wait(&full[stage], phase, err, 29);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t majors = ((A_MN ? 1u : 0u) << 15) | ((B_MN ? 1u : 0u) << 16);
      const uint32_t idesc128 = idesc_bf16_f32(BM, BN) | majors, idesc64 = idesc_bf16_f32(64, BN) | majors;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile ti = decode_tile<SCHED>(args, t);
        if (ti.num_k == 0) continue;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, err, 22)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        // a row tile of at most 64 valid rows runs M = 64 MMAs (same issue time, about half
        // the energy); its rows land in TMEM lanes 32q + (0..15)
        const uint32_t idesc = (SCHED == kSchedRows && ti.rows_valid <= 64) ? idesc64 : idesc128;
        for (int kb = 0; kb < ti.num_k; ++kb) {
          if (!mbar_wait(&full[stage], phase, err, 23)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = A_MN ? sw128_mnmajor_desc(a_addr + kk * 2048) : sw128_kmajor_desc(a_addr + kk * 32);
            const uint64_t bd = B_MN ? sw128_mnmajor_desc(b_addr + kk * 2048) : sw128_kmajor_desc(b_addr + kk * 32);
            tc_mma_f16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc_commit(done);
      mbar_wait(done, 0, err, 24);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2..5)
    const int quarter = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    int chunk = 0;  // kEpiAddF32: reduce-adds issued by this warp (selects the staging buffer)
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile ti = decode_tile<SCHED>(args, t);
      // the tile row of this thread; M = 64 tiles: lanes 0..15 hold rows 16 quarter + lane and
      // lanes 16..31 stand for rows 64..127 (no data: padding rows, written as zeros where the
      // epilogue writes padding)
      const bool m64 = SCHED == kSchedRows && ti.rows_valid <= 64;
      const int row = m64 ? (lane < 16 ? quarter * 16 + lane : 64 + quarter * 16 + (lane - 16)) : quarter * 32 + lane;
      if (ti.num_k == 0) {
        if (EPI == kEpiAddF32 && args.overwrite) {
          // overwrite mode: an expert with no rows has a zero gradient (no MMA, no TMEM)
          constexpr int NB = NBUF > 0 ? NBUF : 1;
          const int m0 = ti.m_blk * BM + quarter * 32;
          // rows from m_split on belong to the second accumulator (tensor map b1)
          const bool second = args.m_split > 0 && m0 >= args.m_split;
          const CUtensorMap* tc = second ? &tmB1 : &tmC;
          const int mc = second ? m0 - args.m_split : m0;
#pragma unroll 1
          for (int c = 0; c < BN; c += 32) {
            const int n0 = ti.n_blk * BN + c;
            if (m0 >= args.m_out || n0 >= args.n_out) continue;
            uint8_t* stg = sStg + (quarter * NB + chunk % NB) * STG_BYTES;
            if (lane == 0) bulk_wait_read<NB - 1>();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(stg + lane * 128 + j * 16) = make_uint4(0, 0, 0, 0);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(tc, stg, n0, mc, ti.g);
              bulk_commit();
            }
            ++chunk;
          }
        }
        continue;
      }
      if (!mbar_wait(&tfull[acc], acc_phase, err, 25)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      if (EPI == kEpiBf16 && !m64 && quarter * 32 + 32 <= ti.rows_valid) {
        // 32 valid rows: coalesced TMA stores of 32 x 64 boxes staged in shared memory (thread =
        // row, chunk j of its 64 values at j ^ (row & 7): the output map's 128-byte swizzle)
        constexpr int NB = NBUF > 0 ? NBUF : 1;
        const int grow0 = (int)ti.a_row + quarter * 32;
#pragma unroll 1
        for (int c = 0; c < BN; c += 64) {
          uint32_t r0[32], r1[32];
          tmem_ld32(tbase + c, r0);
          tmem_ld32(tbase + c + 32, r1);
          tc_wait_ld();
          const int col0 = ti.n_blk * BN + c;
          if (col0 >= args.n_out) continue;  // the same for the whole warp
          uint8_t* stg = sStg + (quarter * NB + chunk % NB) * STG_BYTES;
          if (lane == 0) bulk_wait_read<NB - 1>();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t* v = j < 4 ? r0 + 8 * j : r1 + 8 * (j - 4);
            *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(pack_bf16(__uint_as_float(v[0]), __uint_as_float(v[1])),
                           pack_bf16(__uint_as_float(v[2]), __uint_as_float(v[3])),
                           pack_bf16(__uint_as_float(v[4]), __uint_as_float(v[5])),
                           pack_bf16(__uint_as_float(v[6]), __uint_as_float(v[7])));
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmC, stg, col0, grow0);
            bulk_commit();
          }
          ++chunk;
        }
      } else if (EPI == kEpiBf16) {
        const bool row_ok = row < ti.rows_valid;
        const int64_t grow = ti.a_row + row;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld32(tbase + c, r);
          tc_wait_ld();
          const int col0 = ti.n_blk * BN + c;
          if (row_ok && col0 < args.n_out) {
            uint4* dst = reinterpret_cast<uint4*>(out + grow * args.ldo + col0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 v;
              v.x = pack_bf16(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
              v.y = pack_bf16(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
              v.z = pack_bf16(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
              v.w = pack_bf16(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
              dst[q] = v;
            }
          }
        }
      } else if (EPI == kEpiSwigluBwd) {
        // g = TMEM columns [0,128) (W_g rows), u = [128,256) (W_u rows) of the tile's 128 H columns
        const bool row_ok = row < ti.rows_valid;
        const int64_t grow = ti.a_row + row;
        const int inter = args.inter;
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(tbase + c, g);
          tmem_ld32(tbase + BN / 2 + c, u);
          tc_wait_ld();
          const int col0 = ti.n_blk * (BN / 2) + c;
          if (col0 >= inter) continue;
          const int64_t hoff = grow * inter + col0;
          uint4* dgo = reinterpret_cast<uint4*>(args.dgu + grow * 2 * inter + col0);
          uint4* duo = reinterpret_cast<uint4*>(args.dgu + grow * 2 * inter + inter + col0);
          uint4* ho = reinterpret_cast<uint4*>(args.hpad + hoff);
          const uint4* dhi = reinterpret_cast<const uint4*>(args.dh + hoff);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 vdg = make_uint4(0, 0, 0, 0), vdu = vdg, vh = vdg;
            if (row_ok) {
              const uint4 dh8 = dhi[q];
              const uint32_t dhw[4] = {dh8.x, dh8.y, dh8.z, dh8.w};
              uint32_t* pdg = &vdg.x;
              uint32_t* pdu = &vdu.x;
              uint32_t* ph = &vh.x;
#pragma unroll
              for (int w = 0; w < 4; ++w) {
                const float2 dh2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dhw[w]));
                float da[2], db[2], hv[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const float gv = __uint_as_float(g[8 * q + 2 * w + e]), uv = __uint_as_float(u[8 * q + 2 * w + e]);
                  const float dhv = e ? dh2.y : dh2.x;
                  const float sg = __fdividef(1.0f, 1.0f + __expf(-gv));
                  da[e] = dhv * uv * sg * (1.0f + gv * (1.0f - sg));
                  db[e] = dhv * gv * sg;
                  hv[e] = silu_mul(gv, uv);
                }
                pdg[w] = pack_bf16(da[0], da[1]);
                pdu[w] = pack_bf16(db[0], db[1]);
                ph[w] = pack_bf16(hv[0], hv[1]);
              }
            }
            // rows past the expert's pairs get zeros (weight gradients sum over whole row blocks)
            dgo[q] = vdg;
            duo[q] = vdu;
            ho[q] = vh;
          }
        }
      } else if (EPI == kEpiSwigluSaved) {
        // the accumulator is dH (fp32, 256 columns); g and u are the forward's saved values.
        // The padded rows of an expert's block are its own, so the warp's 32 rows (zeros past
        // the valid ones) leave as 32 x 32 boxes of dG, dU and H by TMA stores (no swizzle;
        // tmC: [dG | dU], tmB1: H), except in M = 64 tiles, whose lanes hold rows of two groups.
        const bool row_ok = row < ti.rows_valid;
        const int64_t grow = ti.a_row + row;
        const int inter = args.inter;
        const bool tma_out = !m64;
        constexpr int NB = NBUF > 0 ? NBUF : 1;
        uint8_t* stg = sStg + quarter * NB * STG_BYTES;  // dG +0, dU +2 KB, H +4 KB
        const int grow0 = (int)ti.a_row + quarter * 32;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld32(tbase + c, r);
          tc_wait_ld();
          const int col0 = ti.n_blk * BN + c;
          if (col0 >= inter) continue;
          if (tma_out) {
            if (lane == 0) bulk_wait_read<0>();  // the previous boxes have been read out
            __syncwarp();
          }
          const uint4* gi = reinterpret_cast<const uint4*>(args.gu + grow * 2 * inter + col0);
          const uint4* ui = reinterpret_cast<const uint4*>(args.gu + grow * 2 * inter + inter + col0);
          uint4* dgo = reinterpret_cast<uint4*>(args.dgu + grow * 2 * inter + col0);
          uint4* duo = reinterpret_cast<uint4*>(args.dgu + grow * 2 * inter + inter + col0);
          uint4* ho = reinterpret_cast<uint4*>(args.hpad + grow * inter + col0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 vdg = make_uint4(0, 0, 0, 0), vdu = vdg, vh = vdg;
            if (row_ok) {
              const uint4 g8 = gi[q], u8 = ui[q];
              const uint32_t gw[4] = {g8.x, g8.y, g8.z, g8.w}, uw[4] = {u8.x, u8.y, u8.z, u8.w};
              uint32_t* pdg = &vdg.x;
              uint32_t* pdu = &vdu.x;
              uint32_t* ph = &vh.x;
#pragma unroll
              for (int w = 0; w < 4; ++w) {
                const float2 g2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[w]));
                const float2 u2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uw[w]));
                float da[2], db[2], hv[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const float gv = e ? g2.y : g2.x, uv = e ? u2.y : u2.x;
                  const float dhv = __uint_as_float(r[8 * q + 2 * w + e]);
                  const float sg = __fdividef(1.0f, 1.0f + __expf(-gv));
                  da[e] = dhv * uv * sg * (1.0f + gv * (1.0f - sg));
                  db[e] = dhv * gv * sg;
                  hv[e] = silu_mul(gv, uv);
                }
                pdg[w] = pack_bf16(da[0], da[1]);
                pdu[w] = pack_bf16(db[0], db[1]);
                ph[w] = pack_bf16(hv[0], hv[1]);
              }
            }
            if (tma_out) {
              *reinterpret_cast<uint4*>(stg + lane * 64 + q * 16) = vdg;
              *reinterpret_cast<uint4*>(stg + 2048 + lane * 64 + q * 16) = vdu;
              *reinterpret_cast<uint4*>(stg + 4096 + lane * 64 + q * 16) = vh;
            } else {
              dgo[q] = vdg;
              duo[q] = vdu;
              ho[q] = vh;
            }
          }
          if (tma_out) {
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmC, stg, col0, grow0);
              tma_store_2d(&tmC, stg + 2048, inter + col0, grow0);
              tma_store_2d(&tmB1, stg + 4096, col0, grow0);
              bulk_commit();
            }
          }
        }
      } else {
        // fused GemmAdd: acc[g][m][n] += product in fp32, done by TMA reduce-adds of
        // 32 x 32 boxes (the L2 does the read-modify-write; each element is added once);
        // overwrite mode: TMA stores of the same boxes (acc[g][m][n] = product).  With m_split,
        // one launch serves two accumulators (dW_g and dW_u over [dG | dU]): rows from m_split
        // on go to the second one (tensor map b1) at row - m_split
        const int m0 = ti.m_blk * BM + quarter * 32;
        const bool second = args.m_split > 0 && m0 >= args.m_split;
        const CUtensorMap* tc = second ? &tmB1 : &tmC;
        const int mc = second ? m0 - args.m_split : m0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld32(tbase + c, r);
          tc_wait_ld();
          const int n0 = ti.n_blk * BN + c;
          if (m0 >= args.m_out || n0 >= args.n_out) continue;
          constexpr int NB = NBUF > 0 ? NBUF : 1;  // (NBUF is 0 in the instantiations without GemmAdd)
          uint8_t* stg = sStg + (quarter * NB + chunk % NB) * STG_BYTES;
          if (lane == 0) bulk_wait_read<NB - 1>();  // the reduce NB chunks back has read this buffer
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (args.overwrite) tma_store_3d(tc, stg, n0, mc, ti.g);
            else tma_reduce_add_3d(tc, stg, n0, mc, ti.g);
            bulk_commit();
          }
          ++chunk;
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if ((EPI == kEpiAddF32 || EPI == kEpiBf16 || EPI == kEpiSwigluSaved) && lane == 0)
      bulk_wait_all();  // every store complete before exit
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int SCHED, bool A_MN, bool B_MN, int EPI>
cudaError_t launch_variant(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const CUtensorMap& c,
                           const BwdArgs& args, int grid, cudaStream_t s) {
  static SmemAttr attr{};
  const cudaError_t e = ensure_smem_attr(attr, k_bwd_gemm<SCHED, A_MN, B_MN, EPI>, Cfg<EPI>::kSmem);
  if (e != cudaSuccess) return e;
  k_bwd_gemm<SCHED, A_MN, B_MN, EPI><<<grid, NUM_THREADS, Cfg<EPI>::kSmem, s>>>(a, b0, b1, c, args);
  return cudaGetLastError();
}

}  // namespace

int bwd_smem_bytes() { return Cfg<kEpiAddF32>::kSmem > Cfg<kEpiBf16>::kSmem ? Cfg<kEpiAddF32>::kSmem : Cfg<kEpiBf16>::kSmem; }

cudaError_t launch_bwd_gemm(int kind, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                            const CUtensorMap& c, const BwdArgs& args, int grid, cudaStream_t s) {
  switch (kind) {
    case kBwdRowsMnB:  // dH, dX, router dx: A K-major, B MN-major, bf16 out
      return launch_variant<kSchedRows, false, true, kEpiBf16>(a, b0, b1, c, args, grid, s);
    case kBwdSwiglu:  // gate/up recompute + SwiGLU backward
      return launch_variant<kSchedRows, false, false, kEpiSwigluBwd>(a, b0, b1, c, args, grid, s);
    case kBwdWgrad:  // weight gradients, fused GemmAdd
      return launch_variant<kSchedWgrad, true, true, kEpiAddF32>(a, b0, b1, c, args, grid, s);
    case kBwdDhSwiglu:  // dH = dY W_d with the SwiGLU backward on the forward's saved G, U
      return launch_variant<kSchedRows, false, true, kEpiSwigluSaved>(a, b0, b1, c, args, grid, s);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace zc
