// Grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM, operands staged by TMA).
//
// One persistent kernel serves the three dense contractions of the layer:
//   router : logits[T, E]        = x[T, d] . W_r[E, d]^T (+ per-expert logit offset), fp32 out
//   gate/up: H[p, inter]         = silu(X_e W_g,e^T) * (X_e W_u,e^T) for the rows p of expert e, bf16 out
//            (training: also G and U themselves, rounded to bf16, for the backward)
//   down   : Y[p, d]             = H_e W_d,e^T, bf16 out
// (LongCat-Flash technical summary, zhangjingwei.cn, 二 架構 / 模型配置: each FFN
// expert is 2048 wide on a 6144 hidden size; the per-expert GEMMs run as one
// grouped GEMM, 五 訓練基礎設施 "優化的分組GEMM", 六 推理與部署 "MoEGEMM".)
//
// Tile: 128 rows (tokens) x 256 columns x 64-deep k-blocks, bf16 operands in
// 128-byte-swizzled K-major shared-memory tiles, fp32 accumulators in TMEM
// (two 256-column buffers, so the epilogue of one tile overlaps the MMAs of
// the next).  For gate/up the 256 B rows are 128 rows of W_g followed by the
// same 128 rows of W_u, so each thread of the epilogue holds the gate and up
// value of the same (row, column) and applies SwiGLU before one bf16 rounding.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues the MMAs (one thread), warps 2..5 drain TMEM (thread = row).
// Tiles are walked expert-major, then column tile, then row block, so the row
// blocks that share a weight tile run on neighbouring SMs at the same time and
// a weight tile is fetched from HBM about once; an expert's activation rows
// stay in L2 across its column tiles.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zc_internal.h"
#include "zc_ptx.cuh"

namespace zc {
namespace {

constexpr int BM = kBM, BN = 256, BK = 64, STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;
constexpr uint32_t B_BYTES = BN * BK * 2;
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr uint32_t STG_BYTES = 32 * 128;  // down epilogue: a 32-row x 64-column bf16 box per warp and buffer
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 4 * 2 * STG_BYTES + 256;

struct Tile {
  int a_row;       // first A row of the tile
  int rows_valid;  // rows of the tile that belong to it
  int b_row;       // first B row
  int n_blk;       // output column tile
  int p_row;       // grouped modes: the tile's first row in the padded layout (128 (mb_off[g] + row block))
};

template <int MODE>
__device__ __forceinline__ int total_tiles(const TcArgs& a) {
  if (MODE == kRouter) return ((a.M + BM - 1) / BM) * a.nblocks;
  return a.mb_off[a.ngroups] * a.nblocks;
}

template <int MODE>
__device__ __forceinline__ Tile decode_tile(const TcArgs& a, int t) {
  Tile ti;
  if (MODE == kRouter) {
    const int m_blk = t / a.nblocks;
    ti.n_blk = t - m_blk * a.nblocks;
    ti.a_row = m_blk * BM;
    ti.rows_valid = min(BM, a.M - ti.a_row);
    ti.b_row = ti.n_blk * BN;
    ti.p_row = ti.a_row;
    return ti;
  }
  // largest expert g with mb_off[g] * nblocks <= t (it has at least one row block)
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
  ti.n_blk = local / nmb;
  const int m_blk = local - ti.n_blk * nmb;
  const int r0 = a.row_off[g];
  ti.a_row = r0 + m_blk * BM;
  ti.rows_valid = min(BM, a.row_off[g + 1] - ti.a_row);
  ti.p_row = (mb0 + m_blk) * BM;
  ti.b_row = g * a.b_rows_per_group + ti.n_blk * (MODE == kGateUp ? BN / 2 : BN);
  return ti;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// TMA store of one staged box (128-byte swizzled in shared memory) at (x, y); completion
// tracked as a bulk group of this thread.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tm, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
              const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmC, const TcArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sStg = sB + STAGES * B_BYTES;  // 1024-aligned: [warp quarter][buffer] of STG_BYTES
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + 4 * 2 * STG_BYTES);
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

  const int total = total_tiles<MODE>(args);
  const int num_k = (args.K + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int fills = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile ti = decode_tile<MODE>(args, t);
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, err, 1)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = sA + stage * A_BYTES;
          uint8_t* b_dst = sB + stage * B_BYTES;
          mbar_expect_tx(&full[stage], STAGE_BYTES);
          tma_load_2d(a_dst, &tmA, kb * BK, ti.a_row, &full[stage]);
          if (MODE == kGateUp) {
            tma_load_2d(b_dst, &tmB0, kb * BK, ti.b_row, &full[stage]);
            tma_load_2d(b_dst + B_BYTES / 2, &tmB1, kb * BK, ti.b_row, &full[stage]);
          } else {
            tma_load_2d(b_dst, &tmB0, kb * BK, ti.b_row, &full[stage]);
          }
          ++fills;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // No TMA write may still be in flight when the CTA exits: wait for the
      // last fills of every stage to land (they already have on the normal path).
      const int pending = fills < STAGES ? fills : STAGES;
      for (int i = 0; i < pending; ++i) {
        if (--stage < 0) {
          stage = STAGES - 1;
          phase ^= 1u;
        }
        mbar_wait(&full[stage], phase, err, 9);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc128 = idesc_bf16_f32(BM, BN);
      constexpr uint32_t idesc64 = idesc_bf16_f32(64, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, err, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        // a tile of at most 64 valid rows (an expert's last row block) runs M = 64 MMAs: the
        // same issue time as M = 128, about half the energy (a power-capped GPU keeps a higher
        // clock); its rows land in TMEM lanes 32q + (0..15), q = 0..3
        const uint32_t idesc = decode_tile<MODE>(args, t).rows_valid <= 64 ? idesc64 : idesc128;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&full[stage], phase, err, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            tc_mma_f16(d_tmem, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), idesc,
                       (kb | kk) != 0 ? 1u : 0u);
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
      // every MMA of this CTA has completed before TMEM is released
      tc_commit(done);
      mbar_wait(done, 0, err, 4);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter+32)
    int acc = 0;
    uint32_t acc_phase = 0;
    int chunk = 0;  // down: boxes stored by this warp (selects the staging buffer)
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile ti = decode_tile<MODE>(args, t);
      if (!mbar_wait(&tfull[acc], acc_phase, err, 5)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      // M = 64 tiles (see the MMA issuer): row 16 quarter + lane in lanes 0..15 of the quarter
      const bool m64 = ti.rows_valid <= 64;
      const int row_in_tile = m64 ? (lane < 16 ? quarter * 16 + lane : BM) : quarter * 32 + lane;
      const bool row_ok = row_in_tile < ti.rows_valid;
      const int64_t grow = (int64_t)ti.a_row + row_in_tile;
      if (MODE == kGateUp) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(tbase + c, g);
          tmem_ld32(tbase + BN / 2 + c, u);
          tc_wait_ld();
          const int col0 = ti.n_blk * (BN / 2) + c;
          if (row_ok && col0 < args.n_out) {
            uint4* dst = reinterpret_cast<uint4*>(out + grow * args.ldo + col0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 v;
              v.x = pack_bf16(silu_mul(__uint_as_float(g[8 * q + 0]), __uint_as_float(u[8 * q + 0])),
                              silu_mul(__uint_as_float(g[8 * q + 1]), __uint_as_float(u[8 * q + 1])));
              v.y = pack_bf16(silu_mul(__uint_as_float(g[8 * q + 2]), __uint_as_float(u[8 * q + 2])),
                              silu_mul(__uint_as_float(g[8 * q + 3]), __uint_as_float(u[8 * q + 3])));
              v.z = pack_bf16(silu_mul(__uint_as_float(g[8 * q + 4]), __uint_as_float(u[8 * q + 4])),
                              silu_mul(__uint_as_float(g[8 * q + 5]), __uint_as_float(u[8 * q + 5])));
              v.w = pack_bf16(silu_mul(__uint_as_float(g[8 * q + 6]), __uint_as_float(u[8 * q + 6])),
                              silu_mul(__uint_as_float(g[8 * q + 7]), __uint_as_float(u[8 * q + 7])));
              dst[q] = v;
            }
            if (args.gu_save) {
              // training: the pre-activations for the backward, in the padded row layout
              __nv_bfloat16* gs = static_cast<__nv_bfloat16*>(args.gu_save) +
                                  ((int64_t)ti.p_row + row_in_tile) * 2 * args.n_out + col0;
              uint4* gdst = reinterpret_cast<uint4*>(gs);
              uint4* udst = reinterpret_cast<uint4*>(gs + args.n_out);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                gdst[q] = make_uint4(pack_bf16(__uint_as_float(g[8 * q + 0]), __uint_as_float(g[8 * q + 1])),
                                     pack_bf16(__uint_as_float(g[8 * q + 2]), __uint_as_float(g[8 * q + 3])),
                                     pack_bf16(__uint_as_float(g[8 * q + 4]), __uint_as_float(g[8 * q + 5])),
                                     pack_bf16(__uint_as_float(g[8 * q + 6]), __uint_as_float(g[8 * q + 7])));
                udst[q] = make_uint4(pack_bf16(__uint_as_float(u[8 * q + 0]), __uint_as_float(u[8 * q + 1])),
                                     pack_bf16(__uint_as_float(u[8 * q + 2]), __uint_as_float(u[8 * q + 3])),
                                     pack_bf16(__uint_as_float(u[8 * q + 4]), __uint_as_float(u[8 * q + 5])),
                                     pack_bf16(__uint_as_float(u[8 * q + 6]), __uint_as_float(u[8 * q + 7])));
              }
            }
          }
        }
      } else if (MODE == kDown && !m64 && quarter * 32 + 32 <= ti.rows_valid) {
        // 32 valid rows: coalesced TMA stores of 32 x 64 boxes staged in shared memory (thread
        // = row, its 64 bf16 values as eight 16-byte chunks, chunk j at j ^ (row & 7): the
        // 128-byte swizzle of the output tensor map)
        const int grow0 = ti.a_row + quarter * 32;
#pragma unroll 1
        for (int c = 0; c < BN; c += 64) {
          uint32_t r0[32], r1[32];
          tmem_ld32(tbase + c, r0);
          tmem_ld32(tbase + c + 32, r1);
          tc_wait_ld();
          const int col0 = ti.n_blk * BN + c;
          if (col0 >= args.n_out) continue;  // the same for the whole warp
          uint8_t* stg = sStg + (quarter * 2 + (chunk & 1)) * STG_BYTES;
          if (lane == 0) bulk_wait_read_1();  // the store two boxes back has read this buffer
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
      } else if (MODE == kDown) {
        // a partly valid row group (the rows past it belong to the next expert): row stores
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
      } else {
        float* out = static_cast<float*>(args.out);
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld32(tbase + c, r);
          tc_wait_ld();
          const int col0 = ti.n_blk * BN + c;
          if (row_ok && col0 < args.n_out) {
            float* dst = out + grow * args.ldo + col0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (col0 + i < args.n_out) {
                const float add = args.col_add ? args.col_add[col0 + i] : 0.0f;
                dst[i] = __fadd_rn(__uint_as_float(r[i]), add);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
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

template <int MODE>
cudaError_t launch_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const CUtensorMap& c,
                        const TcArgs& args, int grid, cudaStream_t s) {
  static SmemAttr attr{};
  const cudaError_t e = ensure_smem_attr(attr, k_tc_gemm<MODE>, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  k_tc_gemm<MODE><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(a, b0, b1, c, args);
  return cudaGetLastError();
}

}  // namespace

int tc_smem_bytes() { return SMEM_BYTES; }
int tc_block_n(int mode) { return mode == kGateUp ? BN / 2 : BN; }

cudaError_t launch_tc_gemm(int mode, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                           const CUtensorMap& c, const TcArgs& args, int grid, cudaStream_t s) {
  switch (mode) {
    case kRouter:
      return launch_mode<kRouter>(a, b0, b1, c, args, grid, s);
    case kGateUp:
      return launch_mode<kGateUp>(a, b0, b1, c, args, grid, s);
    case kDown:
      return launch_mode<kDown>(a, b0, b1, c, args, grid, s);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace zc
