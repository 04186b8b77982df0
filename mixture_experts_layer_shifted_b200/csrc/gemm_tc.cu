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
// Row blocks of 128 tokens x 256 columns x 64-deep k-blocks, bf16 operands in
// 128-byte-swizzled K-major shared-memory tiles, fp32 accumulators in TMEM (two
// 256-column slots).  For gate/up the 256 B rows are 128 rows of W_g followed by
// the same 128 rows of W_u, so each thread of the epilogue holds the gate and up
// value of the same (row, column) and applies SwiGLU before one bf16 rounding.
//
// Work unit of the grouped modes: one weight tile (an expert's 256 B rows) and
// up to TWO of that expert's row blocks.  Each k-block stages the weight tile
// once and both row blocks' activations, and the MMAs of both row blocks read
// the same staged weights, so every SM keeps twice the distinct weight bytes in
// flight that one row block per tile would (the expert GEMMs stream 38.6 GB of
// weights at about 255 tokens per expert, where HBM latency, not the tensor
// pipe, paced the one-row-block schedule).  A pair fills both TMEM slots; a
// single row block (an expert's odd last block, or every router tile) takes one,
// so consecutive singles still overlap the epilogue of one with the MMAs of the
// next.
//
// Scheduling: units are numbered expert-major, then column tile, then row-block
// pair, and handed out by an atomic counter (pairs cost twice a single, and a
// static round-robin over the mixed costs left some SMs with 20% more work).
// Neighbouring units share weight tiles through L2, and an expert's activation
// rows stay in L2 across its column tiles.  The unit ids travel from the
// producer to the MMA and epilogue warps through a small ring in shared memory.
//
// Warp roles (320 threads): warp 0 takes units and issues TMA loads, warp 1 owns
// TMEM and issues the MMAs (one elected lane of the converged warp), warps 2..9
// drain TMEM: two warps per TMEM sub-partition, thread = row, each warp of a
// pair taking half the columns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zc_internal.h"
#include "zc_ptx.cuh"

namespace zc {
namespace {

constexpr int BM = kBM, BN = 256, BK = 64;
constexpr uint32_t A_BYTES = BM * BK * 2;
constexpr int EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr uint32_t STG_BYTES = 32 * 128;  // down epilogue: a 32-row x 64-column bf16 box per warp
constexpr int RING = 4;                   // unit ids in flight from the producer to the consumers
constexpr int BN_NARROW = kRouterNarrowN;

// Columns per tile: 256, or 32 for the narrow router (a batch of one or a few row blocks,
// where 256-column tiles would leave most SMs idle; every logit still sums the same
// K = 16 MMA steps in the same order, so the tile width does not change its value).
template <int MODE>
constexpr int block_n() { return MODE == kRouterNarrow ? BN_NARROW : BN; }

template <int MODE, bool PAIR>
struct Cfg {
  static constexpr bool kPair = PAIR && MODE != kRouter && MODE != kRouterNarrow;  // two row blocks per weight tile
  static constexpr int kBN = block_n<MODE>();
  static constexpr uint32_t kBBytes = kBN * BK * 2;
  static constexpr int kStages = MODE == kRouterNarrow ? 8 : kPair ? 3 : 4;
  static constexpr uint32_t kStageBytes = kBBytes + (kPair ? 2 : 1) * A_BYTES;
  static constexpr uint32_t kTmemCols = 2 * kBN;  // two accumulator slots
  // stages | staging boxes | barriers, the unit ring and the TMEM address
  static constexpr int kSmem = 1024 + kStages * kStageBytes + EPI_WARPS * STG_BYTES + 512;
};

struct Unit {
  int a_row;    // first A row of the first row block
  int rows[2];  // valid rows of each row block (rows[1] = 0: one row block)
  int b_row;    // first B row
  int n_blk;    // output column tile
  int p_row;    // grouped modes: padded-layout row of the first row block (128 (mb_off[g] + block))
  int keep_b;   // 1: an expert's odd last row block beside its pairs -- it streams the same weight tile
                // ahead of them, so its weight lines are loaded with the L2 evict-last priority;
                // 2: a pair of such an expert -- the last reader of those lines, so evict-first
};

template <int MODE, bool PAIR>
__device__ __forceinline__ int total_units(const TcArgs& a) {
  if (MODE == kRouter || MODE == kRouterNarrow) return ((a.M + BM - 1) / BM) * a.nblocks;
  return (PAIR ? a.sp_off[a.ngroups] : a.mb_off[a.ngroups]) * a.nblocks;
}

template <int MODE, bool PAIR>
__device__ __forceinline__ Unit decode_unit(const TcArgs& a, int t) {
  Unit u;
  if (MODE == kRouter || MODE == kRouterNarrow) {
    const int m_blk = t / a.nblocks;
    u.n_blk = t - m_blk * a.nblocks;
    u.a_row = m_blk * BM;
    u.rows[0] = min(BM, a.M - u.a_row);
    u.rows[1] = 0;
    u.b_row = u.n_blk * block_n<MODE>();
    u.keep_b = 0;
    u.p_row = u.a_row;
    return u;
  }
  // units per expert and column tile: its row-block pairs (PAIR) or its row blocks; the
  // largest expert g with off[g] * nblocks <= t (it has at least one unit)
  const int32_t* off = PAIR ? a.sp_off : a.mb_off;
  int lo = 0, hi = a.ngroups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] * a.nblocks <= t) lo = mid;
    else hi = mid - 1;
  }
  const int g = lo;
  const int u0 = off[g];
  const int nu = off[g + 1] - u0;
  const int local = t - u0 * a.nblocks;
  u.n_blk = local / nu;
  const int m0 = (PAIR ? 2 : 1) * (local - u.n_blk * nu);
  const int end = a.row_off[g + 1];
  u.a_row = a.row_off[g] + m0 * BM;
  u.rows[0] = min(BM, end - u.a_row);
  u.rows[1] = PAIR ? max(0, min(BM, end - u.a_row - BM)) : 0;
  u.p_row = (a.mb_off[g] + m0) * BM;
  const int mb = a.mb_off[g + 1] - a.mb_off[g];
  u.keep_b = !PAIR || (mb & 1) == 0 || mb < 3 ? 0 : (u.rows[1] == 0 ? 1 : 2);
  u.b_row = g * a.b_rows_per_group + u.n_blk * (MODE == kGateUp ? BN / 2 : BN);
  return u;
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
__device__ __forceinline__ void bulk_wait_read_0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// The whole warp waits (every lane polls the barrier, bounded); true only if every lane saw it.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* err, int code) {
  const bool ok = mbar_wait(bar, parity, err, code);
  return __all_sync(0xffffffffu, ok);
}

// Epilogue of one row block: warp `quarter` drains TMEM lanes [32 quarter, 32 quarter + 32)
// of the accumulator at tbase; `half` selects which half of the columns this warp takes.
template <int MODE>
__device__ __forceinline__ void drain_rows(const TcArgs& args, const CUtensorMap* tmC, uint32_t tbase, int quarter,
                                           int half, int lane, int a_row, int rows_valid, int p_row, int n_blk,
                                           uint8_t* stg) {
  // an M = 64 accumulator holds row 16 quarter + lane in lanes 0..15 of the quarter
  const bool m64 = rows_valid <= 64;
  const int row_in_tile = m64 ? (lane < 16 ? quarter * 16 + lane : BM) : quarter * 32 + lane;
  const bool row_ok = row_in_tile < rows_valid;
  const int64_t grow = (int64_t)a_row + row_in_tile;
  if (MODE == kGateUp) {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
#pragma unroll 1
    for (int c = half * (BN / 4); c < (half + 1) * (BN / 4); c += 32) {
      uint32_t g[32], u[32];
      tmem_ld32(tbase + c, g);
      tmem_ld32(tbase + BN / 2 + c, u);
      tc_wait_ld();
      const int col0 = n_blk * (BN / 2) + c;
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
          __nv_bfloat16* gs =
              static_cast<__nv_bfloat16*>(args.gu_save) + ((int64_t)p_row + row_in_tile) * 2 * args.n_out + col0;
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
  } else if (MODE == kDown && !m64 && quarter * 32 + 32 <= rows_valid) {
    // 32 valid rows: coalesced TMA stores of 32 x 64 boxes staged in shared memory (thread
    // = row, its 64 bf16 values as eight 16-byte chunks, chunk j at j ^ (row & 7): the
    // 128-byte swizzle of the output tensor map)
    const int grow0 = a_row + quarter * 32;
#pragma unroll 1
    for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += 64) {
      uint32_t r0[32], r1[32];
      tmem_ld32(tbase + c, r0);
      tmem_ld32(tbase + c + 32, r1);
      tc_wait_ld();
      const int col0 = n_blk * BN + c;
      if (col0 >= args.n_out) continue;  // the same for the whole warp
      if (lane == 0) bulk_wait_read_0();  // the previous store of this warp has read the buffer
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
        tma_store_2d(tmC, stg, col0, grow0);
        bulk_commit();
      }
    }
  } else if (MODE == kDown) {
    // a partly valid row group (the rows past it belong to the next expert): row stores
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
#pragma unroll 1
    for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += 32) {
      uint32_t r[32];
      tmem_ld32(tbase + c, r);
      tc_wait_ld();
      const int col0 = n_blk * BN + c;
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
    // router: fp32 logits (+ the logit offset); a 32-column tile is drained by the first
    // warp of each lane quarter alone
    constexpr int bn = block_n<MODE>();
    constexpr int cw = bn >= 64 ? bn / 2 : bn;
    float* out = static_cast<float*>(args.out);
#pragma unroll 1
    for (int c = half * cw; c < (half + 1) * cw && c < bn; c += 32) {
      uint32_t r[32];
      tmem_ld32(tbase + c, r);
      tc_wait_ld();
      const int col0 = n_blk * bn + c;
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
}

template <int MODE, bool PAIR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
              const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmC, const TcArgs args) {
  using C = Cfg<MODE, PAIR>;
  constexpr int STAGES = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // stage s: [B: 256 x 64][A0: 128 x 64][A1: 128 x 64 (pairs only)], each 1024-aligned
  uint8_t* sStg = smem + STAGES * C::kStageBytes;  // [epilogue warp] of STG_BYTES
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + EPI_WARPS * STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* ufull = tempty + 2;
  uint64_t* uempty = ufull + RING;
  uint64_t* done = uempty + RING;
  volatile int* ring = reinterpret_cast<volatile int*>(done + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(ring) + RING);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = args.err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 32 * EPI_WARPS);
    }
    for (int r = 0; r < RING; ++r) {
      mbar_init(&ufull[r], 1);
      mbar_init(&uempty[r], 1 + EPI_WARPS);  // the MMA warp and every epilogue warp read the id
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
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total = total_units<MODE, C::kPair>(args);
  const int num_k = (args.K + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- scheduler + TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int fills = 0;
      bool ok = true;
      const uint64_t keep_policy = l2_policy_evict_last(), drop_policy = l2_policy_evict_first();
      for (int i = 0; i <= total && ok; ++i) {
        const int rs = i % RING;
        if (!mbar_wait(&uempty[rs], ((i / RING) & 1) ^ 1u, err, 10)) break;
        int t = atomicAdd(args.sched, 1);
        if (t >= total) t = -1;
        ring[rs] = t;
        mbar_arrive(&ufull[rs]);
        if (t < 0) break;
        const Unit u = decode_unit<MODE, C::kPair>(args, t);
        const bool two = C::kPair && u.rows[1] > 0;
        const uint32_t bytes = C::kBBytes + (two ? 2u : 1u) * A_BYTES;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, err, 1)) {
            ok = false;
            break;
          }
          uint8_t* b_dst = smem + stage * C::kStageBytes;
          uint8_t* a_dst = b_dst + C::kBBytes;
          mbar_expect_tx(&full[stage], bytes);
          if (u.keep_b) {
            const uint64_t pol = u.keep_b == 1 ? keep_policy : drop_policy;
            tma_load_2d_hint(b_dst, &tmB0, kb * BK, u.b_row, &full[stage], pol);
            if (MODE == kGateUp) tma_load_2d_hint(b_dst + C::kBBytes / 2, &tmB1, kb * BK, u.b_row, &full[stage], pol);
          } else {
            tma_load_2d(b_dst, &tmB0, kb * BK, u.b_row, &full[stage]);
            if (MODE == kGateUp) tma_load_2d(b_dst + C::kBBytes / 2, &tmB1, kb * BK, u.b_row, &full[stage]);
          }
          tma_load_2d(a_dst, &tmA, kb * BK, u.a_row, &full[stage]);
          if (two) tma_load_2d(a_dst + A_BYTES, &tmA, kb * BK, u.a_row + BM, &full[stage]);
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
    // ---------------------------------------------------------------- MMA issuer (converged warp)
    constexpr uint32_t idesc128 = idesc_bf16_f32(BM, C::kBN);
    constexpr uint32_t idesc64 = idesc_bf16_f32(64, C::kBN);
    int stage = 0;
    uint32_t phase = 0;
    int slot = 0;              // TMEM slot of the next row block
    uint32_t uses[2] = {0, 0};  // row blocks each slot has held so far
    bool ok = true;
    for (int i = 0; i <= total && ok; ++i) {
      const int rs = i % RING;
      if (!warp_wait(&ufull[rs], (i / RING) & 1, err, 11)) break;
      const int t = ring[rs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&uempty[rs]);
      if (t < 0) break;
      const Unit u = decode_unit<MODE, C::kPair>(args, t);
      const bool two = C::kPair && u.rows[1] > 0;
      const int s0 = slot, s1 = slot ^ 1;
      // Each slot's accumulator must have been drained by the epilogue of its previous use.  The
      // epilogue frees a pair's slots in order, s0 first, so a pair's first row block starts on
      // the staged k-blocks as soon as s0 is free; the second row block's MMAs on those k-blocks
      // (which keep their stages until then) follow once s1 is free too.
      if (!warp_wait(&tempty[s0], (uses[s0] & 1) ^ 1u, err, 2)) break;
      tc_fence_after();
      const uint32_t d0 = tmem_base + (uint32_t)(s0 * C::kBN), d1 = tmem_base + (uint32_t)(s1 * C::kBN);
      // a row block of at most 64 valid rows runs M = 64 MMAs (about half the energy of
      // M = 128); its rows land in TMEM lanes 32q + (0..15), q = 0..3
      const uint32_t id0 = u.rows[0] <= 64 ? idesc64 : idesc128;
      const uint32_t id1 = u.rows[1] <= 64 ? idesc64 : idesc128;
      const uint32_t par1 = (uses[s1] & 1) ^ 1u;
      bool ready1 = !two;        // s1 free (or not needed)
      int held = 0;              // leading k-blocks whose second-row-block MMAs wait for s1
      const int stage0 = stage;  // the stage of the unit's first k-block
      // second row block's MMAs of k-block kb staged at st, then release the stage (elected lane)
      auto mma_second = [&](int kb, int st) {
        const uint32_t b_addr = smem_u32(smem + st * C::kStageBytes);
        const uint32_t a_addr = b_addr + C::kBBytes + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          tc_mma_f16(d1, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), id1,
                     (kb | kk) != 0 ? 1u : 0u);
        tc_commit(&empty[st]);
      };
      for (int kb = 0; kb < num_k; ++kb) {
        if (!ready1 && held == STAGES) {  // every stage is held: wait for s1 now
          if (!warp_wait(&tempty[s1], par1, err, 2)) {
            ok = false;
            break;
          }
          ready1 = true;
          tc_fence_after();
          if (elect_one())
            for (int j = 0; j < held; ++j) mma_second(j, (stage0 + j) % STAGES);
          __syncwarp();
          held = 0;
        }
        if (!warp_wait(&full[stage], phase, err, 3)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (!ready1) {
          int r = 0;
          if (lane == 0) r = mbar_poll(&tempty[s1], par1) ? 1 : 0;
          ready1 = __shfl_sync(0xffffffffu, r, 0) != 0;
          if (ready1) tc_fence_after();
        }
        if (elect_one()) {
          const uint32_t b_addr = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t a_addr = b_addr + C::kBBytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_f16(d0, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), id0,
                       (kb | kk) != 0 ? 1u : 0u);
          if (!two) {
            tc_commit(&empty[stage]);
          } else if (ready1) {
            for (int j = 0; j < held; ++j) mma_second(j, (stage0 + j) % STAGES);
            mma_second(kb, stage);
          }
        }
        __syncwarp();
        if (two) held = ready1 ? 0 : held + 1;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && !ready1) {  // a unit shorter than the held stages: s1 before the accumulators close
        if (!warp_wait(&tempty[s1], par1, err, 2)) break;
        tc_fence_after();
        if (elect_one())
          for (int j = 0; j < held; ++j) mma_second(j, (stage0 + j) % STAGES);
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) {
        tc_commit(&tfull[s0]);
        if (two) tc_commit(&tfull[s1]);
      }
      __syncwarp();
      ++uses[s0];
      if (two) ++uses[s1];
      else slot ^= 1;
    }
    // every MMA of this CTA has completed before TMEM is released
    if (elect_one()) tc_commit(done);
    __syncwarp();
    warp_wait(done, 0, err, 4);
  } else {
    // ---------------------------------------------------------------- epilogue (8 warps)
    const int quarter = warp & 3;           // TMEM lanes [32 quarter, 32 quarter + 32)
    const int half = (warp - 2) >> 2;       // which half of the columns
    uint8_t* stg = sStg + (warp - 2) * STG_BYTES;
    int slot = 0;
    uint32_t uses[2] = {0, 0};
    bool ok = true;
    for (int i = 0; i <= total && ok; ++i) {
      const int rs = i % RING;
      if (!warp_wait(&ufull[rs], (i / RING) & 1, err, 12)) break;
      const int t = ring[rs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&uempty[rs]);
      if (t < 0) break;
      const Unit u = decode_unit<MODE, C::kPair>(args, t);
      const int nrb = (C::kPair && u.rows[1] > 0) ? 2 : 1;
      for (int r = 0; r < nrb; ++r) {
        const int s = slot ^ r;
        if (!warp_wait(&tfull[s], uses[s] & 1, err, 5)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(s * C::kBN);
        drain_rows<MODE>(args, &tmC, tbase, quarter, half, lane, u.a_row + r * BM, u.rows[r], u.p_row + r * BM,
                         u.n_blk, stg);
        tc_fence_before();
        mbar_arrive(&tempty[s]);
        ++uses[s];
      }
      if (nrb == 1) slot ^= 1;
    }
    if (MODE == kDown && lane == 0) bulk_wait_all();  // every store complete before exit
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <int MODE, bool PAIR>
cudaError_t launch_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const CUtensorMap& c,
                        const TcArgs& args, int grid, cudaStream_t s) {
  using C = Cfg<MODE, PAIR>;
  static SmemAttr attr{};
  cudaError_t e = ensure_smem_attr(attr, k_tc_gemm<MODE, PAIR>, C::kSmem);
  if (e != cudaSuccess) return e;
  if (!args.sched || (C::kPair && !args.sp_off)) return cudaErrorInvalidValue;
  e = cudaMemsetAsync(args.sched, 0, sizeof(int), s);  // the scheduler's unit counter starts at 0
  if (e != cudaSuccess) return e;
  k_tc_gemm<MODE, PAIR><<<grid, NUM_THREADS, C::kSmem, s>>>(a, b0, b1, c, args);
  return cudaGetLastError();
}

}  // namespace

int tc_smem_bytes() {
  return Cfg<kGateUp, true>::kSmem > Cfg<kGateUp, false>::kSmem ? Cfg<kGateUp, true>::kSmem
                                                                : Cfg<kGateUp, false>::kSmem;
}
int tc_block_n(int mode) { return mode == kGateUp ? BN / 2 : mode == kRouterNarrow ? BN_NARROW : BN; }

cudaError_t launch_tc_gemm(int mode, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                           const CUtensorMap& c, const TcArgs& args, int grid, cudaStream_t s) {
  switch (mode) {
    case kRouter:
      return launch_mode<kRouter, false>(a, b0, b1, c, args, grid, s);
    case kRouterNarrow:
      return launch_mode<kRouterNarrow, false>(a, b0, b1, c, args, grid, s);
    case kGateUp:
      return args.pair ? launch_mode<kGateUp, true>(a, b0, b1, c, args, grid, s)
                       : launch_mode<kGateUp, false>(a, b0, b1, c, args, grid, s);
    case kDown:
      return args.pair ? launch_mode<kDown, true>(a, b0, b1, c, args, grid, s)
                       : launch_mode<kDown, false>(a, b0, b1, c, args, grid, s);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace zc
