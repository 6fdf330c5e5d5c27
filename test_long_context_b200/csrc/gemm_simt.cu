// fp32 SIMT GEMM (the TTT_F32 mode: plain FFMA, no TF32, so that fp32 parity
// at 1e-4 relative holds).  Same operand conventions and epilogues as the
// tensor-core GEMM; tile 64 x 128 x 16, 256 threads, 4 x 8 outputs each:
// rows ty*4+i, columns tx*4+j and 64+tx*4+j (so a SwiGLU gate column and its
// up column land in the same thread).  The k-slices of both tiles sit in
// shared memory with the row (m or n) contiguous, each row padded by 4
// floats: a thread reads its 4 A values and its two groups of 4 B values as
// three 16-byte loads, and the transposing stores of K-major operands (16
// lanes on one m or n) spread over banks instead of piling onto one.
#include "gemm.cuh"

namespace ttt {
namespace {

constexpr int SBM = 64, SBN = 128, SBK = 16;
constexpr int SPAD = 4;  // row padding (floats): keeps 16-byte alignment, breaks the stores' bank pile-up

template <bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const float* __restrict__ A, int64_t lda,
                                                        const float* __restrict__ B, int64_t ldb, int64_t M,
                                                        int64_t N, int64_t K, EpiArgs ep) {
  __shared__ __align__(16) float As[SBK][SBM + SPAD];
  __shared__ __align__(16) float Bs[SBK][SBN + SPAD];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = (int64_t)blockIdx.y * SBM, n0 = (int64_t)blockIdx.x * SBN;
  float acc[4][8] = {};
  for (int64_t k0 = 0; k0 < K; k0 += SBK) {
    for (int e = tid; e < SBK * SBM; e += 256) {
      int kk, mm;
      if (A_MN) { kk = e / SBM; mm = e % SBM; } else { mm = e / SBK; kk = e % SBK; }
      const int64_t m = m0 + mm, k = k0 + kk;
      float v = 0.f;
      if (m < M && k < K) v = A_MN ? A[k * lda + m] : A[m * lda + k];
      As[kk][mm] = v;
    }
    for (int e = tid; e < SBK * SBN; e += 256) {
      int kk, nn;
      if (B_MN) { kk = e / SBN; nn = e % SBN; } else { nn = e / SBK; kk = e % SBK; }
      const int64_t n = n0 + nn, k = k0 + kk;
      float v = 0.f;
      if (n < N && k < K) v = B_MN ? B[k * ldb + n] : B[n * ldb + k];
      Bs[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SBK; ++kk) {
      const float4 av = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][64 + tx * 4]);
      const float a[4] = {av.x, av.y, av.z, av.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

  auto col_of = [&](int j) -> int64_t { return n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4)); };

  if constexpr (EPI == EPI_CE_FWD) {
    // one partial (max, sum exp) per row and 128-column tile; 16 lanes share a row group
    for (int i = 0; i < 4; ++i) {
      const int64_t row = m0 + ty * 4 + i;
      const bool row_ok = row < M;
      const int64_t tgt = row_ok ? (int64_t)ep.row_i[row] - ep.col_offset : -1;
      float mx = -INFINITY;
      for (int j = 0; j < 8; ++j)
        if (col_of(j) < N) mx = fmaxf(mx, acc[i][j]);
      for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float sm = 0.f;
      for (int j = 0; j < 8; ++j)
        if (col_of(j) < N) sm += expf(acc[i][j] - mx);
      for (int o = 8; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
      if (row_ok) {
        for (int j = 0; j < 8; ++j)
          if (col_of(j) == tgt) ep.target_logit[row] = acc[i][j];
        if (tx == 0) {
          ep.part_max[(int64_t)blockIdx.x * ep.part_ld + row] = mx;
          ep.part_sum[(int64_t)blockIdx.x * ep.part_ld + row] = sm;
        }
      }
    }
    return;
  }

  for (int i = 0; i < 4; ++i) {
    const int64_t row = m0 + ty * 4 + i;
    if (row >= M) continue;
    if constexpr (EPI == EPI_SWIGLU) {
      for (int j = 0; j < 4; ++j) {
        const int64_t cg = n0 + tx * 4 + j, cu = cg + 64;
        if (cu >= N) continue;
        const float g = acc[i][j], u = acc[i][4 + j];
        if (ep.c2) {
          float* raw = reinterpret_cast<float*>(ep.c2) + row * ep.ldc2;
          raw[cg] = g;
          raw[cu] = u;
        }
        reinterpret_cast<float*>(ep.c)[row * ep.ldc + n0 / 2 + tx * 4 + j] = g / (1.f + expf(-g)) * u;
      }
    } else {
      for (int j = 0; j < 8; ++j) {
        const int64_t col = col_of(j);
        if (col >= N) continue;
        const float v = acc[i][j];
        if constexpr (EPI == EPI_STORE_F32) {
          reinterpret_cast<float*>(ep.c)[row * ep.ldc + col] = v;
        } else if constexpr (EPI == EPI_STORE_BF16) {
          reinterpret_cast<bf16*>(ep.c)[row * ep.ldc + col] = __float2bfloat16_rn(v);
        } else if constexpr (EPI == EPI_ADD_F32) {
          const float r = ep.c2 ? reinterpret_cast<const float*>(ep.c2)[row * ep.ldc2 + col]
                                : reinterpret_cast<float*>(ep.c)[row * ep.ldc + col];
          reinterpret_cast<float*>(ep.c)[row * ep.ldc + col] = r + v;
        } else if constexpr (EPI == EPI_CE_BWD) {
          const float p = expf(v - ep.row_f[row]);
          const float onehot = (col + ep.col_offset == (int64_t)ep.row_i[row]) ? 1.f : 0.f;
          reinterpret_cast<float*>(ep.c)[row * ep.ldc + col] = (p - onehot) * ep.row_g[row];
        } else if constexpr (EPI == EPI_SGD) {
          float* w = reinterpret_cast<float*>(ep.c) + row * ep.ldc + col;
          const float nw = *w - ep.alpha * v;
          *w = nw;
          if (ep.c2) reinterpret_cast<float*>(ep.c2)[row * ep.ldc2 + col] = nw;
        }
      }
    }
  }
}

using SimtFn = void (*)(const float*, int64_t, const float*, int64_t, int64_t, int64_t, int64_t, EpiArgs);

template <bool A_MN, bool B_MN>
SimtFn simt_pick(int epi) {
  switch (epi) {
    case EPI_STORE_F32: return &simt_gemm_kernel<A_MN, B_MN, EPI_STORE_F32>;
    case EPI_STORE_BF16: return &simt_gemm_kernel<A_MN, B_MN, EPI_STORE_BF16>;
    case EPI_ADD_F32: return &simt_gemm_kernel<A_MN, B_MN, EPI_ADD_F32>;
    case EPI_SWIGLU: return &simt_gemm_kernel<A_MN, B_MN, EPI_SWIGLU>;
    case EPI_CE_FWD: return &simt_gemm_kernel<A_MN, B_MN, EPI_CE_FWD>;
    case EPI_CE_BWD: return &simt_gemm_kernel<A_MN, B_MN, EPI_CE_BWD>;
    case EPI_SGD: return &simt_gemm_kernel<A_MN, B_MN, EPI_SGD>;
  }
  return nullptr;
}

}  // namespace

int simt_gemm(const GemmShape& s, int epi, const EpiArgs& args, cudaStream_t stream) {
  const int64_t M = s.M(), N = s.N(), K = s.K();
  if (M < 1 || N < 1 || K < 1 || s.KB() != K) return set_error(TTT_ERR_INVALID_ARG, "gemm: inconsistent shapes");
  if (epi == EPI_SWIGLU && (N % 128) != 0) return set_error(TTT_ERR_INVALID_ARG, "gemm: SwiGLU needs N % 128 == 0");
  SimtFn fn = nullptr;
  if (!s.a_mn && !s.b_mn) fn = simt_pick<false, false>(epi);
  else if (!s.a_mn && s.b_mn) fn = simt_pick<false, true>(epi);
  else if (s.a_mn && s.b_mn) fn = simt_pick<true, true>(epi);
  else fn = simt_pick<true, false>(epi);
  if (!fn) return set_error(TTT_ERR_INVALID_ARG, "gemm: bad epilogue");
  dim3 grid(ceil_div(N, SBN), ceil_div(M, SBM));
  fn<<<grid, 256, 0, stream>>>(reinterpret_cast<const float*>(s.a.ptr), s.a.ld,
                               reinterpret_cast<const float*>(s.b.ptr), s.b.ld, M, N, K, args);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

}  // namespace ttt
