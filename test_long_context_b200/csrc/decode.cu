// Greedy-generation kernels (decode.cuh): one position per step, so every
// product is a matrix-vector product and every kernel streams its operands
// from HBM once.
//
// gemv_kernel: 8 warps per block, x staged in shared memory, one warp per
// output row (two rows - gate and up - for the SwiGLU epilogue); each lane
// reads 16-byte vectors of its row, four of them in flight, with the
// evict-first hint (weights are read once per step); fp32 accumulation and
// a butterfly sum over the warp.  The grid is capped at 8 blocks per SM and
// walks the rows; the LM-head variant keeps, per warp, the running maximum,
// the lowest row attaining it and the sum of exponentials relative to it,
// and writes one partial per block for argmax_finalize.
//
// attn_decode_kernel: grid (head, split of 128 keys); thread t scores key t
// of the split against the query (16-byte loads of its key row), the block
// forms exp(s - m) for its keys, then threads in (group, column pair) layout
// accumulate P V over the split's value rows (each value row read as one
// coalesced line per group).  The last split of a head to finish (a counter
// per head in the work space) merges the splits' (max, sum, o) into o and the
// log-sum-exp, so one launch does the whole product.
#include <algorithm>

#include "decode.cuh"

namespace ttt {
namespace {

constexpr int GV_WARPS = 8;
constexpr int GV_THREADS = 32 * GV_WARPS;
constexpr int GV_MAX_BLOCKS = 148 * 8;

template <typename T>
struct VecOf;
template <>
struct VecOf<bf16> {
  static constexpr int N = 8;
};
template <>
struct VecOf<float> {
  static constexpr int N = 4;
};

__device__ __forceinline__ float dot16(const uint4& w, const uint4& x, float acc, bf16) {
  const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(&w);
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 fa = __bfloat1622float2(a[i]), fb = __bfloat1622float2(b[i]);
    acc = fmaf(fa.x, fb.x, acc);
    acc = fmaf(fa.y, fb.y, acc);
  }
  return acc;
}
__device__ __forceinline__ float dot16(const uint4& w, const uint4& x, float acc, float) {
  acc = fmaf(__uint_as_float(w.x), __uint_as_float(x.x), acc);
  acc = fmaf(__uint_as_float(w.y), __uint_as_float(x.y), acc);
  acc = fmaf(__uint_as_float(w.z), __uint_as_float(x.z), acc);
  acc = fmaf(__uint_as_float(w.w), __uint_as_float(x.w), acc);
  return acc;
}

// o[e] += w * x[e] over the elements of 16 bytes of x
__device__ __forceinline__ void axpy16(float w, const uint4& x, float (&o)[8], bf16) {
  const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(a[i]);
    o[2 * i] = fmaf(w, f.x, o[2 * i]);
    o[2 * i + 1] = fmaf(w, f.y, o[2 * i + 1]);
  }
}
__device__ __forceinline__ void axpy16(float w, const uint4& x, float (&o)[4], float) {
  o[0] = fmaf(w, __uint_as_float(x.x), o[0]);
  o[1] = fmaf(w, __uint_as_float(x.y), o[1]);
  o[2] = fmaf(w, __uint_as_float(x.z), o[2]);
  o[3] = fmaf(w, __uint_as_float(x.w), o[3]);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// W[row, :] . x over k elements (x in shared memory); every lane gets the sum.
template <typename T>
__device__ __forceinline__ float row_dot(const T* __restrict__ w, const T* xs, int64_t k, int lane) {
  constexpr int V = VecOf<T>::N;
  constexpr int64_t STEP = 32 * V;
  const uint4* wv = reinterpret_cast<const uint4*>(w);
  const uint4* xv = reinterpret_cast<const uint4*>(xs);
  const int64_t nv = k / V;  // 16-byte vectors in the row
  float acc0 = 0.f, acc1 = 0.f;
  int64_t i = lane;
  for (; i + 96 < nv; i += 128) {  // four vectors per lane in flight
    const uint4 a0 = __ldcs(wv + i), a1 = __ldcs(wv + i + 32), a2 = __ldcs(wv + i + 64), a3 = __ldcs(wv + i + 96);
    acc0 = dot16(a0, xv[i], acc0, T());
    acc1 = dot16(a1, xv[i + 32], acc1, T());
    acc0 = dot16(a2, xv[i + 64], acc0, T());
    acc1 = dot16(a3, xv[i + 96], acc1, T());
  }
  for (; i < nv; i += 32) acc0 = dot16(__ldcs(wv + i), xv[i], acc0, T());
  (void)STEP;
  return warp_sum(acc0 + acc1);
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.f + __expf(-g)) * u; }

// Running (max, lowest row with the max, sum of exp(y - max)).
struct ArgMax {
  float m = -INFINITY, s = 0.f;
  int64_t i = INT64_MAX;
  __device__ __forceinline__ void add(float y, int64_t r) {
    if (y > m) {
      s = s * expf(m - y) + 1.f;
      m = y;
      i = r;
    } else if (y == m) {
      s += 1.f;
      i = r < i ? r : i;
    } else {
      s += expf(y - m);
    }
  }
  __device__ __forceinline__ void merge(float m2, float s2, int64_t i2) {
    if (m2 == -INFINITY) return;
    if (m2 > m) {
      s = s * expf(m - m2) + s2;
      m = m2;
      i = i2;
    } else if (m2 == m) {
      s += s2;
      i = i2 < i ? i2 : i;
    } else {
      s += s2 * expf(m2 - m);
    }
  }
};

template <typename T, int EPI>
__global__ void __launch_bounds__(GV_THREADS) gemv_kernel(GemvArgs<T> a) {
  extern __shared__ __align__(16) uint8_t gv_smem[];
  constexpr int V = VecOf<T>::N;
  T* xs = reinterpret_cast<T*>(gv_smem);
  T* xs2 = a.x2 ? xs + a.k : xs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (a.xres) {
    // RMSNorm of the residual row, in every block (the same order everywhere)
    __shared__ float nred[GV_WARPS];
    const float4* x4 = reinterpret_cast<const float4*>(a.xres);
    float ss = 0.f;
    for (int64_t i = threadIdx.x; i < a.k / 4; i += GV_THREADS) {
      const float4 v = x4[i];
      ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
    ss = warp_sum(ss);
    if (lane == 0) nred[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < GV_WARPS; ++w) tot += nred[w];
    const float r = 1.f / sqrtf(tot / (float)a.k + a.eps);
    const float4* g4 = reinterpret_cast<const float4*>(a.gain);
    for (int64_t i = threadIdx.x; i < a.k / 4; i += GV_THREADS) {
      const float4 v = x4[i], gg = g4[i];
      const T y0 = from_f32<T>(v.x * r * gg.x), y1 = from_f32<T>(v.y * r * gg.y);
      const T y2 = from_f32<T>(v.z * r * gg.z), y3 = from_f32<T>(v.w * r * gg.w);
      xs[4 * i] = y0;
      xs[4 * i + 1] = y1;
      xs[4 * i + 2] = y2;
      xs[4 * i + 3] = y3;
      if (blockIdx.x == 0 && a.h_out) {
        a.h_out[4 * i] = y0;
        a.h_out[4 * i + 1] = y1;
        a.h_out[4 * i + 2] = y2;
        a.h_out[4 * i + 3] = y3;
      }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0 && a.r_out) *a.r_out = r;
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(a.x);
    uint4* dst = reinterpret_cast<uint4*>(xs);
    for (int64_t i = threadIdx.x; i < a.k / V; i += GV_THREADS) dst[i] = src[i];
  }
  if (a.w2 && a.x2) {
    const uint4* src2 = reinterpret_cast<const uint4*>(a.x2);
    uint4* dst2 = reinterpret_cast<uint4*>(xs2);
    for (int64_t i = threadIdx.x; i < a.k2 / V; i += GV_THREADS) dst2[i] = src2[i];
  }
  __syncthreads();
  const int64_t units = EPI == GEMV_SWIGLU ? a.n / 2 : a.n;
  ArgMax am;
  for (int64_t u = (int64_t)blockIdx.x * GV_WARPS + warp; u < units; u += (int64_t)gridDim.x * GV_WARPS) {
    if constexpr (EPI == GEMV_SWIGLU) {
      const int64_t rg = (u / 64) * 128 + (u % 64), ru = rg + 64;
      float g = row_dot(a.w + rg * a.ldw, xs, a.k, lane);
      float up = row_dot(a.w + ru * a.ldw, xs, a.k, lane);
      if (rg >= a.n_ext) {
        g += row_dot(a.w2 + (rg - a.n_ext) * a.ldw2, xs2, a.k2, lane);
        up += row_dot(a.w2 + (ru - a.n_ext) * a.ldw2, xs2, a.k2, lane);
      }
      if (lane == 0) {
        reinterpret_cast<T*>(a.out)[u] = from_f32<T>(silu_mul(g, up));
        if (a.raw) {
          a.raw[rg] = from_f32<T>(g);
          a.raw[ru] = from_f32<T>(up);
        }
      }
    } else {
      float y = row_dot(a.w + u * a.ldw, xs, a.k, lane);
      if (u >= a.n_ext) y += row_dot(a.w2 + (u - a.n_ext) * a.ldw2, xs2, a.k2, lane);
      if constexpr (EPI == GEMV_STORE) {
        if (lane == 0) reinterpret_cast<T*>(a.out)[u] = from_f32<T>(y);
      } else if constexpr (EPI == GEMV_ADD_F32) {
        if (lane == 0) reinterpret_cast<float*>(a.out)[u] = a.res[u] + y;
      } else {
        am.add(y, u);  // identical in every lane
      }
    }
  }
  if constexpr (EPI == GEMV_ARGMAX) {
    __shared__ float wm[GV_WARPS], wsum[GV_WARPS];
    __shared__ int64_t wi[GV_WARPS];
    if (lane == 0) {
      wm[warp] = am.m;
      wsum[warp] = am.s;
      wi[warp] = am.i;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      ArgMax b;
      for (int w = 0; w < GV_WARPS; ++w) b.merge(wm[w], wsum[w], wi[w]);
      float* p = a.part + 3 * (int64_t)blockIdx.x;
      p[0] = b.m;
      p[1] = __int_as_float(b.i == INT64_MAX ? -1 : (int)b.i);
      p[2] = b.s;
    }
  }
}

__global__ void __launch_bounds__(1024) argmax_finalize_kernel(const float* part, int64_t nparts, int32_t* tok_out,
                                                               int32_t* tgt_row, float* lse_row, float* loss_out) {
  __shared__ float sm[1024], ss[1024];
  __shared__ int64_t si[1024];
  ArgMax am;
  for (int64_t b = threadIdx.x; b < nparts; b += 1024) {
    const int idx = __float_as_int(part[3 * b + 1]);
    if (idx >= 0) am.merge(part[3 * b], part[3 * b + 2], idx);
  }
  sm[threadIdx.x] = am.m;
  ss[threadIdx.x] = am.s;
  si[threadIdx.x] = am.i;
  __syncthreads();
  for (int w = 512; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) {
      ArgMax x;
      x.m = sm[threadIdx.x];
      x.s = ss[threadIdx.x];
      x.i = si[threadIdx.x];
      x.merge(sm[threadIdx.x + w], ss[threadIdx.x + w], si[threadIdx.x + w]);
      sm[threadIdx.x] = x.m;
      ss[threadIdx.x] = x.s;
      si[threadIdx.x] = x.i;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int32_t tok = (int32_t)si[0];
    const float lse = sm[0] + logf(ss[0]);
    *tok_out = tok;
    if (tgt_row) *tgt_row = tok;
    if (lse_row) *lse_row = lse;
    if (loss_out) *loss_out = lse - sm[0];
  }
}

constexpr int AD_KEYS = 128;  // keys per split = threads per block

template <typename T, int HD>
__global__ void __launch_bounds__(AD_KEYS) attn_decode_kernel(const T* q, const T* kr, const T* vr, int64_t ldkv,
                                                              int64_t R, int64_t p, int64_t jlo, float scale,
                                                              float* ws, unsigned* counters, int nsplit, T* o_out,
                                                              float* lse_out, int64_t ld_lse) {
  constexpr int V = VecOf<T>::N;
  constexpr int CV = HD / V;             // 16-byte column vectors of a head row
  constexpr int GROUPS = AD_KEYS / CV;   // key groups of the P V phase
  constexpr int NKT = (AD_KEYS + GROUPS - 1) / GROUPS;  // keys per thread in the P V phase
  constexpr int NKT_PRE = NKT <= 16 ? NKT : 0;          // prefetched into registers when few
  const int h = blockIdx.x, sp = blockIdx.y, t = threadIdx.x;
  __shared__ __align__(16) T qs[HD];
  __shared__ float ps[AD_KEYS];
  __shared__ float red[AD_KEYS / 32];
  __shared__ float oacc[GROUPS][HD];
  if (t < HD) qs[t] = q[(int64_t)h * HD + t];
  __syncthreads();
  const int64_t j0 = jlo + (int64_t)sp * AD_KEYS;
  const int nk = (int)imin64(AD_KEYS, p - j0 + 1);
  // P V layout: thread (g, c) sums column vector c (16 bytes) over keys g, g + GROUPS, ...
  const int g = t / CV, c = t % CV;
  const T* vbase = vr + (int64_t)h * HD + c * V;
  float s = -INFINITY;
  uint4 kk[CV];
  if (t < nk) {
    const uint4* kv = reinterpret_cast<const uint4*>(kr + ((j0 + t) % R) * ldkv + (int64_t)h * HD);
#pragma unroll
    for (int i = 0; i < CV; ++i) kk[i] = __ldcs(kv + i);  // all loads of the key row in flight
  }
  // the value rows of this thread's keys, requested together with the key rows
  uint4 vpre[NKT_PRE > 0 ? NKT_PRE : 1];
  if constexpr (NKT_PRE > 0) {
    if (g < GROUPS) {
#pragma unroll
      for (int u = 0; u < NKT_PRE; ++u) {
        const int kv2 = g + u * GROUPS;
        if (kv2 < nk) vpre[u] = __ldcs(reinterpret_cast<const uint4*>(vbase + ((j0 + kv2) % R) * ldkv));
      }
    }
  }
  if (t < nk) {
    const uint4* qv = reinterpret_cast<const uint4*>(qs);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < CV; ++i) acc = dot16(kk[i], qv[i], acc, T());
    s = acc * scale;
  }
  // block max
  float m = s;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((t & 31) == 0) red[t >> 5] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int w = 1; w < AD_KEYS / 32; ++w) m = fmaxf(m, red[w]);
  const float pt = t < nk ? expf(s - m) : 0.f;
  ps[t] = pt;
  float l = warp_sum(pt);
  __syncthreads();  // every warp has read red[] for the max
  if ((t & 31) == 0) red[t >> 5] = l;
  __syncthreads();
  l = 0.f;
#pragma unroll
  for (int w = 0; w < AD_KEYS / 32; ++w) l += red[w];
  // P V over this thread's keys: from the prefetched value rows, or (long rows
  // of fp32 heads) four value rows in flight at a time
  float o[V];
#pragma unroll
  for (int e = 0; e < V; ++e) o[e] = 0.f;
  if constexpr (NKT_PRE > 0) {
    if (g < GROUPS) {
#pragma unroll
      for (int u = 0; u < NKT_PRE; ++u) {
        const int kv2 = g + u * GROUPS;
        if (kv2 < nk) axpy16(ps[kv2], vpre[u], o, T());
      }
#pragma unroll
      for (int e = 0; e < V; ++e) oacc[g][c * V + e] = o[e];
    }
  } else if (g < GROUPS) {
    int kk = g;
    for (; kk + 3 * GROUPS < nk; kk += 4 * GROUPS) {
      uint4 v4[4];
      float w4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v4[u] = __ldcs(reinterpret_cast<const uint4*>(vbase + ((j0 + kk + u * GROUPS) % R) * ldkv));
        w4[u] = ps[kk + u * GROUPS];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) axpy16(w4[u], v4[u], o, T());
    }
    for (; kk < nk; kk += GROUPS)
      axpy16(ps[kk], __ldcs(reinterpret_cast<const uint4*>(vbase + ((j0 + kk) % R) * ldkv)), o, T());
#pragma unroll
    for (int e = 0; e < V; ++e) oacc[g][c * V + e] = o[e];
  }
  __syncthreads();
  float* out = ws + ((int64_t)h * nsplit + sp) * (HD + 2);
  if (t < HD) {
    float v = 0.f;
#pragma unroll
    for (int gg = 0; gg < GROUPS; ++gg) v += oacc[gg][t];
    out[2 + t] = v;
  }
  if (t == 0) {
    out[0] = m;
    out[1] = l;
  }
  // the last split of this head to finish merges all of them (its counter
  // then returns to zero for the next call)
  __shared__ unsigned last;
  __threadfence();
  __syncthreads();
  if (t == 0) last = atomicAdd(&counters[h], 1u) == (unsigned)(nsplit - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  const float* base = ws + (int64_t)h * nsplit * (HD + 2);
  __shared__ float sf[AD_KEYS + 1];  // per-split factor exp(m_s - M); [AD_KEYS] = L
  float ms = -INFINITY;
  if (t < nsplit) ms = __ldcg(base + (int64_t)t * (HD + 2));
  float M = ms;
#pragma unroll
  for (int o2 = 16; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
  if ((t & 31) == 0) red[t >> 5] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int w = 1; w < AD_KEYS / 32; ++w) M = fmaxf(M, red[w]);
  const float fct = t < nsplit ? expf(ms - M) : 0.f;
  sf[t] = fct;
  float lsum = warp_sum(t < nsplit ? __ldcg(base + (int64_t)t * (HD + 2) + 1) * fct : 0.f);
  __syncthreads();
  if ((t & 31) == 0) red[t >> 5] = lsum;
  __syncthreads();
  if (t == 0) {
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < AD_KEYS / 32; ++w) L += red[w];
    sf[AD_KEYS] = L;
  }
  __syncthreads();
  const float L = sf[AD_KEYS];
  if (t < HD) {
    float acc = 0.f;
#pragma unroll 8
    for (int s2 = 0; s2 < nsplit; ++s2) acc = fmaf(__ldcg(base + (int64_t)s2 * (HD + 2) + 2 + t), sf[s2], acc);
    o_out[(int64_t)h * HD + t] = from_f32<T>(acc / L);
  }
  if (t == 0) {
    if (lse_out) lse_out[(int64_t)h * ld_lse] = M + logf(L);
    counters[h] = 0u;
  }
}

__global__ void fill_kernel(float* dst, int64_t n, float v) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = v;
}

template <typename T, int HD>
int launch_attn(const T* q, const T* kr, const T* vr, int64_t ldkv, int64_t R, int H, int64_t p, int64_t window,
                float scale, T* o, float* lse, int64_t ld_lse, float* ws, cudaStream_t s) {
  const int64_t jlo = p - window + 1 > 0 ? p - window + 1 : 0;
  const int nsplit = (int)((p - jlo + AD_KEYS) / AD_KEYS);
  if (nsplit > AD_KEYS) return set_error(TTT_ERR_UNSUPPORTED, "attn_decode: window above 16 384 keys");
  // per-head split counters after the partials (zero between calls)
  unsigned* counters = reinterpret_cast<unsigned*>(ws + (int64_t)H * ((window + AD_KEYS - 1) / AD_KEYS + 1) * (HD + 2));
  attn_decode_kernel<T, HD><<<dim3(H, nsplit), AD_KEYS, 0, s>>>(q, kr, vr, ldkv, R, p, jlo, scale, ws, counters,
                                                                 nsplit, o, lse, ld_lse);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

}  // namespace

int64_t gemv_parts(int64_t n) { return std::min<int64_t>(GV_MAX_BLOCKS, (n + GV_WARPS - 1) / GV_WARPS); }

template <typename T>
int gemv(const GemvArgs<T>& a, int epi, cudaStream_t s) {
  constexpr int V = VecOf<T>::N;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (a.n < 1 || a.k < 1 || a.k % V || !al16(a.w) || (a.ldw * (int64_t)sizeof(T)) % 16 || !a.out)
    return set_error(TTT_ERR_INVALID_ARG, "gemv: rows must be 16-byte aligned and k a multiple of 16 bytes");
  if (a.xres ? (!al16(a.xres) || !al16(a.gain) || a.k % 4) : !al16(a.x))
    return set_error(TTT_ERR_INVALID_ARG, "gemv: input vector misaligned");
  if (a.w2 && (a.k2 < 1 || a.k2 % V || !al16(a.w2) || (a.ldw2 * (int64_t)sizeof(T)) % 16 || (a.x2 && !al16(a.x2)) ||
               (!a.x2 && a.k2 != a.k)))
    return set_error(TTT_ERR_INVALID_ARG, "gemv: second product misaligned");
  if (epi == GEMV_SWIGLU && (a.n % 128 || (a.w2 && a.n_ext % 128)))
    return set_error(TTT_ERR_INVALID_ARG, "gemv: SwiGLU rows come in blocks of 128");
  if (epi == GEMV_ARGMAX && (!a.part || a.n > INT32_MAX)) return set_error(TTT_ERR_INVALID_ARG, "gemv: argmax");
  GemvArgs<T> b = a;
  if (!b.w2) b.n_ext = INT64_MAX, b.k2 = 0;
  const int64_t units = epi == GEMV_SWIGLU ? a.n / 2 : a.n;
  const unsigned blocks = (unsigned)(epi == GEMV_ARGMAX ? gemv_parts(a.n)
                                                        : std::min<int64_t>(GV_MAX_BLOCKS, (units + GV_WARPS - 1) / GV_WARPS));
  const size_t smem = (size_t)(a.k + (b.x2 ? b.k2 : 0)) * sizeof(T);
  if (smem > 200 * 1024) return set_error(TTT_ERR_INVALID_ARG, "gemv: input vector too long for shared memory");
  auto go = [&](auto kern) -> int {
    if (smem > 48 * 1024) TTT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    kern<<<blocks, GV_THREADS, smem, s>>>(b);
    TTT_CUDA_TRY(cudaGetLastError());
    return TTT_OK;
  };
  switch (epi) {
    case GEMV_STORE: return go(gemv_kernel<T, GEMV_STORE>);
    case GEMV_ADD_F32: return go(gemv_kernel<T, GEMV_ADD_F32>);
    case GEMV_SWIGLU: return go(gemv_kernel<T, GEMV_SWIGLU>);
    case GEMV_ARGMAX: return go(gemv_kernel<T, GEMV_ARGMAX>);
  }
  return set_error(TTT_ERR_INVALID_ARG, "gemv: bad epilogue");
}

int argmax_finalize(const float* part, int64_t nparts, int32_t* tok_out, int32_t* tgt_row, float* lse_row,
                    float* loss_out, cudaStream_t s) {
  argmax_finalize_kernel<<<1, 1024, 0, s>>>(part, nparts, tok_out, tgt_row, lse_row, loss_out);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

int64_t attn_decode_ws_floats(int H, int HD, int64_t window) {
  return (int64_t)H * ((window + AD_KEYS - 1) / AD_KEYS + 1) * (HD + 2) + H;
}

template <typename T>
int attn_decode(const T* q, const T* kr, const T* vr, int64_t ldkv, int64_t R, int H, int HD, int64_t p,
                int64_t window, float scale, T* o, float* lse, int64_t ld_lse, float* ws, cudaStream_t s) {
  constexpr int V = VecOf<T>::N;
  if ((ldkv * (int64_t)sizeof(T)) % 16 || (reinterpret_cast<uintptr_t>(kr) & 15) || HD % V || p < 0 || window < 1 ||
      R < window)
    return set_error(TTT_ERR_INVALID_ARG, "attn_decode: bad ring layout");
  switch (HD) {
    case 32: return launch_attn<T, 32>(q, kr, vr, ldkv, R, H, p, window, scale, o, lse, ld_lse, ws, s);
    case 64: return launch_attn<T, 64>(q, kr, vr, ldkv, R, H, p, window, scale, o, lse, ld_lse, ws, s);
    case 80: return launch_attn<T, 80>(q, kr, vr, ldkv, R, H, p, window, scale, o, lse, ld_lse, ws, s);
    case 96: return launch_attn<T, 96>(q, kr, vr, ldkv, R, H, p, window, scale, o, lse, ld_lse, ws, s);
    case 128: return launch_attn<T, 128>(q, kr, vr, ldkv, R, H, p, window, scale, o, lse, ld_lse, ws, s);
  }
  return set_error(TTT_ERR_UNSUPPORTED, "attn_decode: head_dim must be 32, 64, 80, 96 or 128");
}

int fill_f32(float* dst, int64_t n, float v, cudaStream_t s) {
  if (n <= 0) return TTT_OK;
  fill_kernel<<<ceil_div(n, 256), 256, 0, s>>>(dst, n, v);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template int gemv<float>(const GemvArgs<float>&, int, cudaStream_t);
template int gemv<bf16>(const GemvArgs<bf16>&, int, cudaStream_t);
template int attn_decode<float>(const float*, const float*, const float*, int64_t, int64_t, int, int, int64_t, int64_t,
                                float, float*, float*, int64_t, float*, cudaStream_t);
template int attn_decode<bf16>(const bf16*, const bf16*, const bf16*, int64_t, int64_t, int, int, int64_t, int64_t,
                               float, bf16*, float*, int64_t, float*, cudaStream_t);

}  // namespace ttt
