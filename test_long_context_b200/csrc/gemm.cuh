// GEMM interface shared by the engine and the op-level entry points.
//
//   acc[m][n] = sum_k A(m, k) * B(n, k)
//
// Operands are row-major matrix views in storage order:
//   A K-major ("a_mn = 0"): [M rows, K cols];  A MN-major: [K rows, M cols]
//   B K-major ("b_mn = 0"): [N rows, K cols];  B MN-major: [K rows, N cols]
// so a forward projection x W^T is (K, K), a data gradient dY W is (K, MN)
// and a weight gradient dY^T X is (MN, MN).
//
// The epilogue consumes the fp32 accumulator tile: see Epi.
#pragma once
#include "common.cuh"

namespace ttt {

enum Epi : int {
  EPI_STORE_F32 = 0,   // C (fp32) = acc
  EPI_STORE_BF16 = 1,  // C (bf16) = acc
  EPI_ADD_F32 = 2,     // C (fp32) = R + acc, R = C2 (fp32) when given, else C itself
  EPI_SWIGLU = 3,      // columns come in (gate 64 | up 64) pairs: C[:, pair*64 + i] = silu(g) * u
                       // (activation dtype); C2 (optional) = raw acc (activation dtype)
  EPI_CE_FWD = 4,      // per row and N tile: part_max, part_sum of exp; target_logit[row] if the
                       // target column (row_i[row] - col_offset) is in this GEMM's columns;
                       // C (fp32, optional, tensor-core path) = acc (the logits)
  EPI_CE_BWD = 5,      // C (activation dtype) = (exp(acc - row_f[row]) - [col + col_offset ==
                       // row_i[row]]) * row_g[row]
  EPI_SGD = 6,         // C (fp32 master) -= alpha * acc; C2 (optional, bf16) = hi = bf16(new master);
                       // C3 (optional, bf16, with C2) = lo = bf16(new master - hi)
  EPI_COUNT = 7
};

struct EpiArgs {
  void* c = nullptr;
  int64_t ldc = 0;
  void* c2 = nullptr;
  int64_t ldc2 = 0;
  const float* row_f = nullptr;
  const float* row_g = nullptr;
  const int32_t* row_i = nullptr;
  float* part_max = nullptr;
  float* part_sum = nullptr;
  float* target_logit = nullptr;
  int64_t part_ld = 0;  // stride between N tiles in part_max/part_sum
  float alpha = 0.f;
  int64_t col_offset = 0;
  int64_t split_stride = 0;  // split-K partials: elements between consecutive splits (EPI_STORE_F32 only)
  void* c3 = nullptr;  // EPI_SGD: low bf16 half of the new master
  int64_t ldc3 = 0;
};

// Row-major matrix view in storage order (element type given by the GEMM).
struct MatView {
  const void* ptr = nullptr;
  int64_t rows = 0, cols = 0, ld = 0;
};

struct GemmShape {
  int a_mn = 0, b_mn = 0;
  MatView a, b;
  int64_t M() const { return a_mn ? a.cols : a.rows; }
  int64_t K() const { return a_mn ? a.rows : a.cols; }
  int64_t N() const { return b_mn ? b.cols : b.rows; }
  int64_t KB() const { return b_mn ? b.rows : b.cols; }
};

// A prepared tensor-core GEMM (bf16 operands): tensor maps are built once
// and the launch only passes them by value.
struct TcGemm {
  alignas(64) CUtensorMap ta;
  alignas(64) CUtensorMap tb;
  int a_mn = 0, b_mn = 0, bn = 256, epi = 0;
  int pair = 0;  // 256 x 256 tiles on CTA pairs (tcgen05 cta_group::2); B tensor maps then hold 128-row boxes
  int64_t M = 0, N = 0, K = 0;
  EpiArgs args;
  int act_bf16 = 1;  // activation dtype of EPI_SWIGLU / EPI_CE_BWD outputs
  // deterministic split-K (ksplit > 1): partials to ws [ksplit][M][N] fp32, then an ordered reduction
  int ksplit = 1;
  int64_t kps = 0;  // k per split (of the concatenated reduction), a multiple of 64
  float* ws = nullptr;
  // second product A2 B2^T, added on output tiles with n0 >= n_ext (K2 = 0: none)
  alignas(64) CUtensorMap ta2;
  alignas(64) CUtensorMap tb2;
  int64_t K2 = 0, n_ext = 0;
};

// Split-K count for an M x N x K GEMM with this epilogue (1 = no split); sets
// *bn_out to the tile width to use when splitting (0 = default).
int64_t tc_split_plan(int64_t M, int64_t N, int64_t K, int epi, int* bn_out);
// Enable split-K on a prepared GEMM: ws must hold ksplit * M * N floats.
int tc_gemm_set_split(TcGemm* g, int64_t ksplit, float* ws);
// Add a second product: acc += A2 B2^T on output tiles with n0 >= n_ext (a
// multiple of the tile width; B2's rows/cols are counted from n_ext).  A2 and
// B2 take the main operands' orientation; A2 has the same M, B2 covers
// N - n_ext outputs, and they share their own reduction length K2.  Call
// before tc_gemm_set_split; split-K then needs n_ext = 0.
int tc_gemm_set_ext(TcGemm* g, const MatView& a2, const MatView& b2, int64_t n_ext);

// Returns TTT_OK or an error code (bad shapes, tensor-map failure).
int tc_gemm_prepare(TcGemm* g, const GemmShape& s, int epi, const EpiArgs& args, int bn_hint = 0);
int tc_gemm_launch(const TcGemm& g, cudaStream_t stream, int* dev_err);

// fp32 SIMT GEMM with the same semantics (all operands fp32).
int simt_gemm(const GemmShape& s, int epi, const EpiArgs& args, cudaStream_t stream);

// Tile width the tensor-core GEMM uses for an M x N output (hint 128/256 forces it).
int tc_pick_bn(int64_t M, int64_t N, int hint);
// Number of N tiles a CE_FWD GEMM writes partials for (tensor-core path).
int64_t tc_ce_tiles(int64_t N, int bn);

}  // namespace ttt
