// Internal interfaces between the C-ABI layer (zcmoe.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace zc {

// Rows of one tensor-core output tile; also the m-block granularity of the
// expert offsets produced by the integer stage.
constexpr int kBM = 128;
// Tokens per block of the integer stage (8 warps x 32 lanes, one token per thread).
constexpr int kChunk = 256;

// Copies msg into the calling thread's zcmoe_last_error() slot (zcmoe.cu).
void set_last_error(const char* msg);

// A kernel's dynamic shared-memory limit is a per-device attribute.  Each kernel
// keeps one SmemAttr: a bit per device ordinal (0..127), set once the attribute has
// been raised on that device.  Threads may race to set it; the attribute call is
// idempotent and the bits are atomic.
struct SmemAttr {
  std::atomic<uint64_t> done[2];
};
template <typename Kernel>
cudaError_t ensure_smem_attr(SmemAttr& a, Kernel* kernel, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  const uint64_t bit = 1ull << (dev & 63);
  std::atomic<uint64_t>& word = a.done[dev >> 6];
  if (word.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  word.fetch_or(bit, std::memory_order_acq_rel);
  return cudaSuccess;
}

// ------------------------------------------------------------- routing (route.cu)
cudaError_t launch_softmax_topk(const float* logits, const float* bias, int T, int E, int k, float scale, int32_t* idx,
                                float* gate, float* scores, int sms, cudaStream_t s);
cudaError_t launch_route_count(const int32_t* idx, int T, int k, int E, int32_t* chunk_cnt, cudaStream_t s);
// sp_off (nullable): [N+1] prefix of the row-block pairs ceil(mb / 2) (the grouped GEMM's work units)
cudaError_t launch_route_scan(int32_t* chunk_cnt, int nchunks, int T, int N, int E, int32_t* counts, int32_t* offsets,
                              int32_t* mb_off, int32_t* scal, int64_t* acc_counts, int64_t* acc_tokens, cudaStream_t s,
                              int32_t* sp_off = nullptr);
// The three integer-stage kernels in one block for T <= route_small_max_tokens() (same results).
int route_small_max_tokens();
cudaError_t launch_route_small(const int32_t* idx, int T, int k, int N, int E, int32_t* counts, int32_t* offsets,
                               int32_t* mb_off, int32_t* scal, int64_t* acc_counts, int64_t* acc_tokens,
                               int32_t* sp_off, int32_t* perm, int32_t* pos, cudaStream_t s);
cudaError_t launch_route_scatter(const int32_t* idx, int T, int k, int N, int E, const int32_t* chunk_base,
                                 int32_t* perm, int32_t* pos, cudaStream_t s);
// X_perm[pos[t, j]] = x[t] for every FFN slot (pos >= 0): the pairs' rows in expert order
cudaError_t launch_scatter_rows(const void* x, int row_bytes, const int32_t* pos, int T, int k, void* xperm, int sms,
                                cudaStream_t s);
// offsets / mb_off non-null: Y rows are padded (FP8 layers), see k_combine.
cudaError_t launch_combine(int bf16, const void* x, const void* Y, const int32_t* idx, const float* gate,
                           const int32_t* pos, int T, int k, int N, int d, void* y, int sms, cudaStream_t s,
                           const int32_t* offsets = nullptr, const int32_t* mb_off = nullptr);
cudaError_t launch_selftest_wait(int* err, uint64_t limit_ns, cudaStream_t s);
cudaError_t launch_single_group(int32_t* row_off, int32_t* mb_off, int T, cudaStream_t s, int32_t* sp_off = nullptr);
cudaError_t launch_update_bias(int64_t* counts, int64_t* tokens, int N, int Z, int k, float kp, float ki, float kd,
                               float decay, float target, const float* b0, float* eta, float* integ, float* eprev,
                               float* bias, cudaStream_t s);

// ------------------------------------------------------------- tensor-core GEMM (gemm_tc.cu)
enum TcMode { kRouter = 0, kGateUp = 1, kDown = 2, kRouterNarrow = 3 };
constexpr int kRouterNarrowN = 32;  // columns per tile of the narrow router (its W_r tensor map's box)

struct TcArgs {
  int K;                    // reduction length (elements)
  int n_out;                // valid output columns
  int nblocks;              // output column tiles
  int ngroups;              // experts (router: 1)
  const int32_t* row_off;   // [ngroups+1] first permuted row of each expert (router: unused)
  const int32_t* mb_off;    // [ngroups+1] first m-block of each expert (router: unused)
  int M;                    // router: token rows
  int b_rows_per_group;     // rows of the B tensor per expert (gate/up: inter, down: d)
  void* out;                // output matrix
  int64_t ldo;              // its row stride (elements)
  const float* col_add;     // router: per-column offset added to the logits (or null)
  void* gu_save;            // gate/up, optional: the fp32 accumulators G and U rounded to bf16, stored as
                            // [G | U] [padded rows, 2 n_out] (expert g's pairs from row 128 mb_off[g] on)
  int* err;                 // device error word (bounded waits)
  // grouped modes: [ngroups+1] first row-block pair of each expert, prefix of ceil(mb / 2)
  // over the experts' row blocks (the unit of work that shares one staged weight tile)
  const int32_t* sp_off;
  int* sched;               // tile counter of the dynamic scheduler, zeroed by the launcher
  int pair;                 // grouped modes: 1 = units of two row blocks (the expected rows per
                            // expert fill two or more blocks), 0 = one row block per unit
};

// Whether the grouped GEMMs should stage two row blocks per weight tile: when an
// expert's rows are expected to fill at least 128 rows (rows = expected rows per
// expert, from the batch size and the routing fan-out, known on the host).
inline int tc_pair_for_rows(int64_t rows) { return rows >= kBM ? 1 : 0; }

int tc_smem_bytes();
int tc_block_n(int mode);
// c: kDown only -- the output as a 2-D bf16 tensor [rows, n_out], box 64 x 32, 128-byte swizzle
// (its full 32-row groups leave by TMA stores); the other modes ignore it.
cudaError_t launch_tc_gemm(int mode, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                           const CUtensorMap& c, const TcArgs& args, int grid, cudaStream_t s);

// ------------------------------------------------------------- block-scaled FP8 (fp8_quant.cu, gemm_fp8.cu)
// atom_groups > 0: scales written as scale atoms with that many atoms per 128
// rows; 0: plain [row blocks, cols/128].
cudaError_t launch_quant_rows(int bf16, const void* src, int64_t rows, int cols, uint8_t* codes, uint8_t* scales,
                              int atom_groups, int sms, cudaStream_t s);
cudaError_t launch_quant_tiles(int bf16, const void* src, int64_t rows, int cols, uint8_t* codes, uint8_t* scales,
                               int atom_groups, cudaStream_t s);
// MXFP4: [1,32] blocks along each row (cols a multiple of 256), codes two per byte;
// atom_groups > 0: scale atoms with that many atoms (128 elements each) per 128 rows.
cudaError_t launch_quant_mx4(int bf16, const void* src, int64_t rows, int cols, uint8_t* codes, uint8_t* scales,
                             int atom_groups, int sms, cudaStream_t s);
// NVFP4: g[m] = the tensor scale of matrix m (nmat matrices of mrows x cols, consecutive);
// rows of src take gvec[r / rows_per_g] (gvec null: g_const)
cudaError_t launch_nv4_global(int bf16, const void* src, int nmat, int64_t mrows, int cols, float* g, cudaStream_t s);
cudaError_t launch_quant_nv4(int bf16, const void* src, int64_t rows, int cols, uint8_t* codes, uint8_t* scales,
                             int atom_groups, const float* gvec, int64_t rows_per_g, float g_const, int sms,
                             cudaStream_t s);
// The FFN pairs' x rows quantized into the padded expert-order operand of the block-scaled
// GEMM, one warp per token: fmt 0 FP8 [1,128], 1 MXFP4 [1,32], 2 NVFP4 [1,16] (g = 1)
cudaError_t launch_scatter_quant(int fmt, const void* x, int d, const int32_t* pos, const int32_t* idx, int T, int k,
                                 const int32_t* offsets, const int32_t* mb_off, uint8_t* codes, uint8_t* scales,
                                 int groups, int sms, cudaStream_t s);
cudaError_t launch_unpad_rows(const void* ypad, int row_bytes, const int32_t* perm, const int32_t* idx,
                              const int32_t* offsets, const int32_t* mb_off, const int32_t* scal, void* out, int sms,
                              cudaStream_t s);

struct Fp8Args {
  int fmt;                 // 0: FP8 E4M3, [1,128]/[128,128] scales; 1: MXFP4, [1,32] scales; 2: NVFP4, [1,16]
  int K;                   // reduction length in elements (FP8: a multiple of 128, MXFP4 / NVFP4: of 256)
  int n_out;               // valid output columns
  int nblocks;             // output column tiles
  int ngroups;             // experts
  const int32_t* row_off;  // [ngroups+1] pair offsets (the counts' exclusive scan)
  const int32_t* mb_off;   // [ngroups+1] row-block offsets: expert g's rows start at padded row 128 mb_off[g]
  int b_rows_per_group;    // rows of the B tensor per expert (gate/up: inter, down: d)
  const uint8_t* sfa;      // A scale atoms
  const uint8_t* sfb0;     // B scale atoms (gate/up: W_g, down: W_d)
  const uint8_t* sfb1;     // gate/up: W_u scale atoms
  int groups_k;            // scale atoms per 128 rows of A and B: FP8 ceil(K / 512), MXFP4 ceil(K / 128),
                           // NVFP4 K / 64
  const float* gsc0;       // NVFP4: the B tensors' fp32 scales per expert (gate/up: W_g, down: W_d)
  const float* gsc1;       // NVFP4 gate/up: W_u's
  void* out;               // gate/up: H codes [padded rows, n_out (FP8) or n_out / 2 (FP4) bytes]; down: Y bf16
  int64_t ldo;             // its row stride (gate/up: bytes; down: elements)
  uint8_t* out_sf;         // gate/up: H scale atoms, out_groups per 128 rows
  int out_groups;
  int* err;                // device error word (bounded waits)
};
int fp8_smem_bytes();
int fp8_block_n(int mode);
// c: kDown only -- the padded output rows [rows, n_out] bf16, box 32 x 32, no swizzle (whole
// 32-row groups leave by TMA stores); kGateUp ignores it.
cudaError_t launch_fp8_gemm(int mode, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                            const CUtensorMap& c, const Fp8Args& args, int grid, cudaStream_t s);

// ------------------------------------------------------------- backward data movement (moe_bwd.cu, route.cu)
cudaError_t launch_router_bwd(const float* logits, int T, int E, int k, float scale, const int32_t* idx,
                              const float* dg, __nv_bfloat16* dl, int ld, int sms, cudaStream_t s);
cudaError_t launch_gather_pad(const void* x, int d, const int32_t* perm, int k, const int32_t* row_off,
                              const int32_t* mb_off, int N, void* xpad, void* dypad, int sms, cudaStream_t s);
cudaError_t launch_combine_bwd(const void* x, const void* dy, const void* Y, const float* gate, const int32_t* pos,
                               const int32_t* idx, const int32_t* offsets, const int32_t* mb_off, int T, int k, int d,
                               void* dypad, float* dg, cudaStream_t s);
cudaError_t launch_final_dx(const void* dy, const void* dxp, const void* dxr, const float* gate, const int32_t* pos,
                            const int32_t* idx, const int32_t* offsets, const int32_t* mb_off, int T, int k, int d,
                            void* dx, cudaStream_t s);

// ------------------------------------------------------------- backward GEMMs (gemm_bwd.cu)
enum BwdSched { kSchedRows = 0, kSchedWgrad = 1 };
enum BwdEpi { kEpiBf16 = 0, kEpiSwigluBwd = 1, kEpiAddF32 = 2, kEpiSwigluSaved = 3 };
enum BwdKind { kBwdRowsMnB = 0, kBwdSwiglu = 1, kBwdWgrad = 2, kBwdDhSwiglu = 3 };

// ------------------------------------------------------------- expert parallelism (ep.cu)
// Row q of s-major segment i (rows [seg_src[i], seg_src[i+1])) <-> row seg_dst[i] + q - seg_src[i].
cudaError_t launch_ep_regroup(const void* src, void* dst, int64_t P, int row_bytes, const int32_t* seg_src,
                              const int32_t* seg_dst, int nseg, int inverse, int sms, cudaStream_t s);

struct BwdArgs {
  int K;                     // kSchedRows: reduction length (a multiple of 64)
  int n_out, nblocks;        // output columns, 256-column tiles
  int m_out, mblocks;        // kSchedWgrad: output rows, 128-row tiles
  int ngroups;               // experts (1 for the router)
  const int32_t* row_off;    // [ngroups+1] pair offsets
  const int32_t* mb_off;     // [ngroups+1] row-block offsets (expert g's rows start at padded row 128 mb_off[g])
  int a_col0;                // first A column (K offset for K-major A, M offset for MN-major A)
  int64_t b_row_per_group;   // B row offset per expert (K-major B: rows; MN-major B: K rows)
  int k_split;               // MN-major B: K rows [0, k_split) from tmB0, the rest from tmB1 (INT_MAX: none)
  void* out;                 // kEpiBf16: bf16 [padded rows, ldo]
  int64_t ldo;
  const __nv_bfloat16* dh;   // kEpiSwigluBwd: dH [padded rows, inter]
  const __nv_bfloat16* gu;   // kEpiSwigluSaved: the forward's [G | U] [padded rows, 2 inter] (dH is the accumulator)
  __nv_bfloat16* dgu;        //   out (both SwiGLU epilogues): [dG | dU] [padded rows, 2 inter]
  __nv_bfloat16* hpad;       //   out: H [padded rows, inter]
  int inter;
  float* acc;                // kEpiAddF32: acc[g][m][n] += product (through the tensor map c)
  int overwrite;             //   1: acc[g][m][n] = product instead (experts with no rows get zeros)
  int64_t acc_ld, acc_group_stride;
  int m_split;               //   > 0: output rows >= m_split go to a second accumulator (tensor map b1) at
                             //   row - m_split (a multiple of 32), so dW_g and dW_u come from one launch
  int* err;                  // device error word (bounded waits)
};
int bwd_smem_bytes();
// c: kBwdWgrad -- the fp32 accumulator as a 3-D tensor [groups][m_out][n_out], box 32 x 32 x 1,
// 128-byte swizzle (the reduce-add target; with m_split, b1 is the second accumulator's map);
// kBwdRowsMnB -- the bf16 output [rows, n_out], box
// 64 x 32, 128-byte swizzle (full 32-row groups leave by TMA stores); kBwdDhSwiglu -- [dG | dU]
// [rows, 2 inter] bf16, box 32 x 32, no swizzle, with H [rows, inter] the same way as b1; other
// kinds ignore it.
cudaError_t launch_bwd_gemm(int kind, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                            const CUtensorMap& c, const BwdArgs& args, int grid, cudaStream_t s);

// ------------------------------------------------------------- fp32 CUDA-core GEMM (gemm_simt.cu)
struct SimtArgs {
  const float* A;
  const float* B0;
  const float* B1;
  int K;
  int n_out;
  int ngroups;
  const int32_t* row_off;
  const int32_t* mb_off;
  int M;
  int b_rows_per_group;
  float* out;
  int64_t ldo;
  const float* col_add;
};
cudaError_t launch_simt_gemm(int mode, const SimtArgs& args, int max_mblocks, cudaStream_t s);

}  // namespace zc
