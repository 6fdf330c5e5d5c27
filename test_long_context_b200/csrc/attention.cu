// Banded causal sliding-window attention (eq. (1) of the reading notes:
// query p sees keys p-k+1 .. p), forward and the backward the updated blocks
// need.  Keys and values are read from a ring of R slots, slot = position
// mod R, so a chunk's queries can see the previous chunks' cached keys.
//
// SIMT kernels (fp32 math, fp32 or bf16 storage): TPR threads share one query
// (or key) row and split head_dim between them; key (or query) tiles are
// staged in shared memory as fp32.
#include "attention.cuh"

#include <functional>

namespace ttt {
namespace {

constexpr int ATT_THREADS = 128;
constexpr int KT = 32;  // keys (forward, dq) or queries (dk/dv) per shared-memory tile

template <int TPR>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---- forward -----------------------------------------------------------------
template <typename T, int HD, int TPR>
__global__ void __launch_bounds__(ATT_THREADS) swa_fwd_simt(SwaArgs a) {
  constexpr int QB = ATT_THREADS / TPR;
  constexpr int E = HD / TPR;
  __shared__ float Ks[KT][HD + 1];
  __shared__ float Vs[KT][HD + 1];
  const int h = blockIdx.y;
  const int qi = threadIdx.x / TPR, part = threadIdx.x % TPR;
  const int64_t i = (int64_t)blockIdx.x * QB + qi;  // local query row
  const bool valid = i < a.n;
  const int64_t p = a.p0 + i;                        // absolute position
  float q[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    q[e] = valid ? to_f32(reinterpret_cast<const T*>(a.q)[i * a.ldq + h * HD + part + TPR * e]) * a.scale : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int64_t pb = a.p0 + (int64_t)blockIdx.x * QB;
  const int64_t pe = imin64(pb + QB, a.p0 + a.n) - 1;  // last query of the block
  const int64_t jlo = imax64(0, pb - a.window + 1);
  const T* kr = reinterpret_cast<const T*>(a.k);
  const T* vr = reinterpret_cast<const T*>(a.v);
  for (int64_t j0 = jlo; j0 <= pe; j0 += KT) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < KT * HD; idx += ATT_THREADS) {
      const int r = idx / HD, c = idx % HD;
      const int64_t j = j0 + r;
      float kv = 0.f, vv = 0.f;
      if (j <= pe) {
        const int64_t slot = j % a.ring;
        kv = to_f32(kr[slot * a.ldkv + h * HD + c]);
        vv = to_f32(vr[slot * a.ldkv + h * HD + c]);
      }
      Ks[r][c] = kv;
      Vs[r][c] = vv;
    }
    __syncthreads();
    float s[KT];
    float tmax = -INFINITY;
#pragma unroll
    for (int r = 0; r < KT; ++r) {
      float d = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) d = fmaf(q[e], Ks[r][part + TPR * e], d);
      d = group_sum<TPR>(d);
      const int64_t j = j0 + r;
      const bool ok = valid && j <= p && j > p - a.window;
      s[r] = ok ? d : -INFINITY;
      tmax = fmaxf(tmax, s[r]);
    }
    if (tmax == -INFINITY) continue;
    if (tmax > m) {
      const float corr = expf(m - tmax);
      l *= corr;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] *= corr;
      m = tmax;
    }
#pragma unroll
    for (int r = 0; r < KT; ++r) {
      const float pr = expf(s[r] - m);
      l += pr;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(pr, Vs[r][part + TPR * e], acc[e]);
    }
  }
  if (valid) {
    const float inv = 1.f / l;
#pragma unroll
    for (int e = 0; e < E; ++e)
      reinterpret_cast<T*>(a.o)[i * a.ldo + h * HD + part + TPR * e] = from_f32<T>(acc[e] * inv);
    if (part == 0) a.lse[(int64_t)h * a.ld_lse + i] = m + logf(l);
  }
}

// ---- backward: D = rowsum(dO * O) ----------------------------------------------
template <typename T, int HD>
__global__ void swa_bwd_dot(SwaArgs a) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t i = idx / a.heads;
  const int h = (int)(idx % a.heads);
  if (i >= a.n) return;
  const T* o = reinterpret_cast<const T*>(a.o) + i * a.ldo + h * HD;
  const T* d = reinterpret_cast<const T*>(a.dout) + i * a.lddo + h * HD;
  float s = 0.f;
  for (int e = 0; e < HD; ++e) s = fmaf(to_f32(o[e]), to_f32(d[e]), s);
  a.D[(int64_t)h * a.ld_lse + i] = s;
}

// ---- backward: dq over the full band ---------------------------------------------
template <typename T, int HD, int TPR>
__global__ void __launch_bounds__(ATT_THREADS) swa_bwd_dq_simt(SwaArgs a) {
  constexpr int QB = ATT_THREADS / TPR;
  constexpr int E = HD / TPR;
  __shared__ float Ks[KT][HD + 1];
  __shared__ float Vs[KT][HD + 1];
  const int h = blockIdx.y;
  const int qi = threadIdx.x / TPR, part = threadIdx.x % TPR;
  const int64_t i = (int64_t)blockIdx.x * QB + qi;
  const bool valid = i < a.n;
  const int64_t p = a.p0 + i;
  float q[E], dO[E], dq[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int c = h * HD + part + TPR * e;
    q[e] = valid ? to_f32(reinterpret_cast<const T*>(a.q)[i * a.ldq + c]) * a.scale : 0.f;
    dO[e] = valid ? to_f32(reinterpret_cast<const T*>(a.dout)[i * a.lddo + c]) : 0.f;
    dq[e] = 0.f;
  }
  const float lse = valid ? a.lse[(int64_t)h * a.ld_lse + i] : 0.f;
  const float Di = valid ? a.D[(int64_t)h * a.ld_lse + i] : 0.f;
  const int64_t pb = a.p0 + (int64_t)blockIdx.x * QB;
  const int64_t pe = imin64(pb + QB, a.p0 + a.n) - 1;
  const int64_t jlo = imax64(0, pb - a.window + 1);
  const T* kr = reinterpret_cast<const T*>(a.k);
  const T* vr = reinterpret_cast<const T*>(a.v);
  for (int64_t j0 = jlo; j0 <= pe; j0 += KT) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < KT * HD; idx += ATT_THREADS) {
      const int r = idx / HD, c = idx % HD;
      const int64_t j = j0 + r;
      float kv = 0.f, vv = 0.f;
      if (j <= pe) {
        const int64_t slot = j % a.ring;
        kv = to_f32(kr[slot * a.ldkv + h * HD + c]);
        vv = to_f32(vr[slot * a.ldkv + h * HD + c]);
      }
      Ks[r][c] = kv;
      Vs[r][c] = vv;
    }
    __syncthreads();
#pragma unroll 2
    for (int r = 0; r < KT; ++r) {
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        s = fmaf(q[e], Ks[r][part + TPR * e], s);
        dp = fmaf(dO[e], Vs[r][part + TPR * e], dp);
      }
      s = group_sum<TPR>(s);
      dp = group_sum<TPR>(dp);
      const int64_t j = j0 + r;
      const bool ok = valid && j <= p && j > p - a.window;
      const float pr = ok ? expf(s - lse) : 0.f;
      const float ds = pr * (dp - Di);
#pragma unroll
      for (int e = 0; e < E; ++e) dq[e] = fmaf(ds, Ks[r][part + TPR * e], dq[e]);
    }
  }
  if (valid) {
#pragma unroll
    for (int e = 0; e < E; ++e)
      reinterpret_cast<T*>(a.dq)[i * a.lddq + h * HD + part + TPR * e] = from_f32<T>(dq[e] * a.scale);
  }
}

// ---- backward: dk, dv for the chunk's own keys ----------------------------------------
template <typename T, int HD, int TPR>
__global__ void __launch_bounds__(ATT_THREADS) swa_bwd_dkdv_simt(SwaArgs a) {
  constexpr int KB = ATT_THREADS / TPR;  // keys per block
  constexpr int E = HD / TPR;
  __shared__ float Qs[KT][HD + 1];
  __shared__ float Ds[KT][HD + 1];
  __shared__ float Ls[KT], DDs[KT];
  const int h = blockIdx.y;
  const int ki = threadIdx.x / TPR, part = threadIdx.x % TPR;
  const int64_t jl = (int64_t)blockIdx.x * KB + ki;  // local key row (= chunk position)
  const bool valid = jl < a.n;
  const int64_t j = a.p0 + jl;
  const T* kr = reinterpret_cast<const T*>(a.k);
  const T* vr = reinterpret_cast<const T*>(a.v);
  float k[E], v[E], dk[E], dv[E];
  const int64_t slot = valid ? j % a.ring : 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int c = h * HD + part + TPR * e;
    k[e] = valid ? to_f32(kr[slot * a.ldkv + c]) : 0.f;
    v[e] = valid ? to_f32(vr[slot * a.ldkv + c]) : 0.f;
    dk[e] = 0.f;
    dv[e] = 0.f;
  }
  const int64_t jb = (int64_t)blockIdx.x * KB;          // first local key of the block
  const int64_t je = imin64(jb + KB, a.n) - 1;    // last local key
  const int64_t ihi = imin64(je + a.window - 1, a.n - 1);
  for (int64_t i0 = jb; i0 <= ihi; i0 += KT) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < KT * HD; idx += ATT_THREADS) {
      const int r = idx / HD, c = idx % HD;
      const int64_t i = i0 + r;
      float qv = 0.f, dv_ = 0.f;
      if (i <= ihi) {
        qv = to_f32(reinterpret_cast<const T*>(a.q)[i * a.ldq + h * HD + c]) * a.scale;
        dv_ = to_f32(reinterpret_cast<const T*>(a.dout)[i * a.lddo + h * HD + c]);
      }
      Qs[r][c] = qv;
      Ds[r][c] = dv_;
    }
    for (int r = threadIdx.x; r < KT; r += ATT_THREADS) {
      const int64_t i = i0 + r;
      Ls[r] = i <= ihi ? a.lse[(int64_t)h * a.ld_lse + i] : 0.f;
      DDs[r] = i <= ihi ? a.D[(int64_t)h * a.ld_lse + i] : 0.f;
    }
    __syncthreads();
#pragma unroll 2
    for (int r = 0; r < KT; ++r) {
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        s = fmaf(Qs[r][part + TPR * e], k[e], s);
        dp = fmaf(Ds[r][part + TPR * e], v[e], dp);
      }
      s = group_sum<TPR>(s);
      dp = group_sum<TPR>(dp);
      const int64_t i = i0 + r;
      const int64_t pq = a.p0 + i;
      const bool ok = valid && i <= ihi && j <= pq && j > pq - a.window;
      const float pr = ok ? expf(s - Ls[r]) : 0.f;
      const float ds = pr * (dp - DDs[r]);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        dv[e] = fmaf(pr, Ds[r][part + TPR * e], dv[e]);
        dk[e] = fmaf(ds, Qs[r][part + TPR * e], dk[e]);  // Qs already carries the scale
      }
    }
  }
  if (valid) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int c = h * HD + part + TPR * e;
      reinterpret_cast<T*>(a.dk)[jl * a.lddkv + c] = from_f32<T>(dk[e]);
      reinterpret_cast<T*>(a.dv)[jl * a.lddkv + c] = from_f32<T>(dv[e]);
    }
  }
}

template <typename T, int HD>
int launch_fwd(const SwaArgs& a, cudaStream_t s) {
  constexpr int TPR = 2;
  dim3 grid(ceil_div(a.n, ATT_THREADS / TPR), a.heads);
  swa_fwd_simt<T, HD, TPR><<<grid, ATT_THREADS, 0, s>>>(a);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <typename T, int HD>
int launch_bwd(const SwaArgs& a, cudaStream_t s, const std::function<int()>& dq_override,
               const std::function<int()>& dkdv_override) {
  swa_bwd_dot<T, HD><<<ceil_div(a.n * a.heads, 256), 256, 0, s>>>(a);
  TTT_CUDA_TRY(cudaGetLastError());
  if (dq_override) {
    const int rc = dq_override();
    if (rc) return rc;
  } else {
    dim3 g1(ceil_div(a.n, ATT_THREADS / 2), a.heads);
    swa_bwd_dq_simt<T, HD, 2><<<g1, ATT_THREADS, 0, s>>>(a);
    TTT_CUDA_TRY(cudaGetLastError());
  }
  if (dkdv_override) return dkdv_override();
  dim3 g2(ceil_div(a.n, ATT_THREADS / 4), a.heads);
  swa_bwd_dkdv_simt<T, HD, 4><<<g2, ATT_THREADS, 0, s>>>(a);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <typename T>
int dispatch_fwd(const SwaArgs& a, cudaStream_t s) {
  switch (a.head_dim) {
    case 32: return launch_fwd<T, 32>(a, s);
    case 64: return launch_fwd<T, 64>(a, s);
    case 80: return launch_fwd<T, 80>(a, s);
    case 96: return launch_fwd<T, 96>(a, s);
    case 128: return launch_fwd<T, 128>(a, s);
  }
  return set_error(TTT_ERR_UNSUPPORTED, "attention: head_dim must be 32, 64, 80, 96 or 128");
}

template <typename T>
int dispatch_bwd(const SwaArgs& a, cudaStream_t s, const std::function<int()>& dq,
                 const std::function<int()>& dkdv) {
  switch (a.head_dim) {
    case 32: return launch_bwd<T, 32>(a, s, dq, dkdv);
    case 64: return launch_bwd<T, 64>(a, s, dq, dkdv);
    case 80: return launch_bwd<T, 80>(a, s, dq, dkdv);
    case 96: return launch_bwd<T, 96>(a, s, dq, dkdv);
    case 128: return launch_bwd<T, 128>(a, s, dq, dkdv);
  }
  return set_error(TTT_ERR_UNSUPPORTED, "attention: head_dim must be 32, 64, 80, 96 or 128");
}

}  // namespace

int swa_forward(const SwaArgs& a, bool use_bf16, cudaStream_t s) {
  if (a.n < 1 || a.window < 1 || a.ring < 1) return set_error(TTT_ERR_INVALID_ARG, "attention: bad sizes");
  return use_bf16 ? dispatch_fwd<bf16>(a, s) : dispatch_fwd<float>(a, s);
}

int swa_backward(const SwaArgs& a, bool use_bf16, cudaStream_t s) {
  if (a.n < 1 || a.window < 1 || a.ring < 1) return set_error(TTT_ERR_INVALID_ARG, "attention: bad sizes");
  return use_bf16 ? dispatch_bwd<bf16>(a, s, {}, {}) : dispatch_bwd<float>(a, s, {}, {});
}

int swa_backward_with_dq(const SwaArgs& a, bool use_bf16, cudaStream_t s, const std::function<int()>& dq,
                         const std::function<int()>& dkdv) {
  if (a.n < 1 || a.window < 1 || a.ring < 1) return set_error(TTT_ERR_INVALID_ARG, "attention: bad sizes");
  return use_bf16 ? dispatch_bwd<bf16>(a, s, dq, dkdv) : dispatch_bwd<float>(a, s, dq, dkdv);
}

}  // namespace ttt
