// Memory-bound kernels of the prefill loop (see elementwise.cuh).  RMSNorm
// uses one 128-thread block per row with float4 access (one warp per row when
// the layout is not vector-aligned); everything else is one thread per
// element or one warp per row.
#include <algorithm>

#include "elementwise.cuh"

namespace ttt {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int ROW_WARPS = 8;  // rows per 256-thread block

template <typename T>
__global__ void embed_kernel(const int32_t* tok, const T* E, int64_t n, int d, int V, float* x, int* err) {
  const int64_t row = (int64_t)blockIdx.x * ROW_WARPS + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= n) return;
  int t = tok[row];
  if (t < 0 || t >= V) {
    if (lane == 0) atomicOr(err, DEV_ERR_BAD_TOKEN);
    t = 0;
  }
  const T* src = E + (int64_t)t * d;
  float* dst = x + row * d;
  for (int c = lane; c < d; c += 32) dst[c] = to_f32(src[c]);
}

template <typename T>
__global__ void rmsnorm_fwd_kernel(const float* x, int64_t ldx, const float* g, float eps, int64_t n, int d, T* y,
                                   int64_t ldy, float* rstd) {
  const int64_t row = (int64_t)blockIdx.x * ROW_WARPS + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= n) return;
  const float* xr = x + row * ldx;
  float ss = 0.f;
  for (int c = lane; c < d; c += 32) ss = fmaf(xr[c], xr[c], ss);
  ss = warp_sum(ss);
  const float r = 1.f / sqrtf(ss / (float)d + eps);
  T* yr = y + row * ldy;
  for (int c = lane; c < d; c += 32) yr[c] = from_f32<T>(xr[c] * r * g[c]);
  if (lane == 0 && rstd) rstd[row] = r;
}

template <typename T>
__global__ void rmsnorm_bwd_kernel(const float* x, int64_t ldx, const float* rstd, const float* g, const float* dy,
                                   int64_t lddy, const float* dres, int64_t ldres, int64_t n, int d, float* dx,
                                   int64_t lddx, T* dx16, int64_t ld16) {
  const int64_t row = (int64_t)blockIdx.x * ROW_WARPS + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= n) return;
  const float r = rstd[row];
  const float* xr = x + row * ldx;
  const float* dyr = dy + row * lddy;
  float dot = 0.f;
  for (int c = lane; c < d; c += 32) dot = fmaf(xr[c] * r, dyr[c] * g[c], dot);
  dot = warp_sum(dot) / (float)d;
  for (int c = lane; c < d; c += 32) {
    const float u = dyr[c] * g[c];
    float v = r * (u - xr[c] * r * dot);
    if (dres) v += dres[row * ldres + c];
    dx[row * lddx + c] = v;
    if (dx16) dx16[row * ld16 + c] = from_f32<T>(v);
  }
}

// Vectorised RMSNorm: one 128-thread block per row, the row held in
// registers as float4 (d <= 4 * 128 * VN), so x is read once and each block
// reduces with 4 warps.  Used when d and every leading dimension are
// multiples of 4 and the pointers are 16-byte (fp32) / 8-byte (bf16) aligned.
constexpr int VT = 128;  // threads per row
constexpr int VN = 8;    // float4 per thread: d <= 4096

__device__ __forceinline__ float block_sum128(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  const float t = (red[0] + red[1]) + (red[2] + red[3]);
  __syncthreads();  // red may be reused by the caller
  return t;
}

template <typename T> __device__ __forceinline__ void store4(T* p, float4 v);
template <> __device__ __forceinline__ void store4<float>(float* p, float4 v) {
  *reinterpret_cast<float4*>(p) = v;
}
template <> __device__ __forceinline__ void store4<bf16>(bf16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

template <typename T>
__global__ void __launch_bounds__(VT) rmsnorm_fwd_vec_kernel(const float* x, int64_t ldx, const float* g, float eps,
                                                             int d, T* y, int64_t ldy, float* rstd) {
  __shared__ float red[4];
  const int64_t row = blockIdx.x;
  const int d4 = d >> 2;
  const float4* xr = reinterpret_cast<const float4*>(x + row * ldx);
  float4 v[VN];
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < VN; ++u) {
    const int c = threadIdx.x + u * VT;
    v[u] = c < d4 ? xr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
    ss = fmaf(v[u].x, v[u].x, fmaf(v[u].y, v[u].y, fmaf(v[u].z, v[u].z, fmaf(v[u].w, v[u].w, ss))));
  }
  ss = block_sum128(ss, red);
  const float r = 1.f / sqrtf(ss / (float)d + eps);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  T* yr = y + row * ldy;
#pragma unroll
  for (int u = 0; u < VN; ++u) {
    const int c = threadIdx.x + u * VT;
    if (c < d4) {
      const float4 gg = g4[c];
      store4<T>(yr + 4 * c, make_float4(v[u].x * r * gg.x, v[u].y * r * gg.y, v[u].z * r * gg.z, v[u].w * r * gg.w));
    }
  }
  if (threadIdx.x == 0 && rstd) rstd[row] = r;
}

template <typename T>
__global__ void __launch_bounds__(VT) rmsnorm_bwd_vec_kernel(const float* x, int64_t ldx, const float* rstd,
                                                             const float* g, const float* dy, int64_t lddy,
                                                             const float* dres, int64_t ldres, int d, float* dx,
                                                             int64_t lddx, T* dx16, int64_t ld16) {
  __shared__ float red[4];
  const int64_t row = blockIdx.x;
  const int d4 = d >> 2;
  const float r = rstd[row];
  const float4* xr = reinterpret_cast<const float4*>(x + row * ldx);
  const float4* dyr = reinterpret_cast<const float4*>(dy + row * lddy);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  float4 xv[VN], uv[VN];  // x and u = dy * g
  float dot = 0.f;
#pragma unroll
  for (int u = 0; u < VN; ++u) {
    const int c = threadIdx.x + u * VT;
    xv[u] = uv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (c < d4) {
      xv[u] = xr[c];
      const float4 dd = dyr[c], gg = g4[c];
      uv[u] = make_float4(dd.x * gg.x, dd.y * gg.y, dd.z * gg.z, dd.w * gg.w);
    }
    dot = fmaf(xv[u].x * r, uv[u].x, fmaf(xv[u].y * r, uv[u].y, fmaf(xv[u].z * r, uv[u].z, fmaf(xv[u].w * r, uv[u].w, dot))));
  }
  dot = block_sum128(dot, red) / (float)d;
  const float rd = r * dot;
#pragma unroll
  for (int u = 0; u < VN; ++u) {
    const int c = threadIdx.x + u * VT;
    if (c < d4) {
      float4 o = make_float4(r * (uv[u].x - xv[u].x * rd), r * (uv[u].y - xv[u].y * rd),
                             r * (uv[u].z - xv[u].z * rd), r * (uv[u].w - xv[u].w * rd));
      if (dres) {
        const float4 e = reinterpret_cast<const float4*>(dres + row * ldres)[c];
        o.x += e.x;
        o.y += e.y;
        o.z += e.z;
        o.w += e.w;
      }
      reinterpret_cast<float4*>(dx + row * lddx)[c] = o;
      if (dx16) store4<T>(dx16 + row * ld16 + 4 * c, o);
    }
  }
}

__host__ __forceinline__ bool al(const void* p, int b) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) % b) == 0; }

// Rotation table of positions p0 .. p0+n-1: tab[i * HD/2 + t] = (cos, sin) of
// (p0 + i) * theta^(-2t/HD), angles in fp64, stored as fp32.
__global__ void rope_table_kernel(float2* tab, int64_t p0, int64_t n, int HD, double theta) {
  const int h2 = HD / 2;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n * h2) return;
  const int64_t i = idx / h2;
  const int t = (int)(idx % h2);
  const double inv = pow(theta, -2.0 * (double)t / (double)HD);
  double sd, cd;
  sincos((double)(p0 + i) * inv, &sd, &cd);
  tab[idx] = make_float2((float)cd, (float)sd);
}

// QK-norm + RoPE forward, one token per block iteration: the token's q and k
// rows are staged in smem with 16-byte loads, four threads share a head (a
// quarter of its rotation pairs each, sums of squares combined by shuffles),
// and the results leave with 16-byte stores; v is copied to the ring with
// 16-byte accesses.  Needs H * HD a multiple of 16 bytes' worth of elements.
constexpr int ROPE_THREADS = 256;

template <typename T>
__global__ void __launch_bounds__(ROPE_THREADS) qknorm_rope_fwd_kernel(
    const T* __restrict__ qkv, int64_t ldqkv, const float* __restrict__ gq, const float* __restrict__ gk, int64_t n,
    int64_t p0, int H, int HD, float eps, const float2* __restrict__ tab, int64_t tab_p0, T* __restrict__ qout,
    int64_t ldq, T* __restrict__ kring, T* __restrict__ vring, int64_t ldkv, int64_t R, float* __restrict__ rq,
    float* __restrict__ rk) {
  extern __shared__ __align__(16) unsigned char rope_smem[];
  T* row = reinterpret_cast<T*>(rope_smem);  // [2 * D]: q | k of one token
  constexpr int EV = 16 / sizeof(T);          // elements per 16-byte vector
  const int D = H * HD, h2 = HD / 2;
  const int per = (h2 + 3) / 4;               // rotation pairs per thread
  const int tasks = ((8 * H + 31) / 32) * 32; // (q or k head, quarter), padded to whole warps
  for (int64_t i = blockIdx.x; i < n; i += gridDim.x) {
    const T* src = qkv + i * ldqkv;
    const int64_t slot = (p0 + i) % R;
    for (int c = threadIdx.x; c < 2 * D / EV; c += blockDim.x)
      reinterpret_cast<uint4*>(row)[c] = reinterpret_cast<const uint4*>(src)[c];
    for (int c = threadIdx.x; c < D / EV; c += blockDim.x)
      reinterpret_cast<uint4*>(vring + slot * ldkv)[c] = reinterpret_cast<const uint4*>(src + 2 * D)[c];
    __syncthreads();
    const float2* cs = tab + (p0 + i - tab_p0) * h2;
    for (int task = threadIdx.x; task < tasks; task += blockDim.x) {
      const int hh = task / 4, part = task % 4;  // hh < H: q head hh; else k head hh - H
      const bool live = hh < 2 * H;
      const int t0 = part * per, t1 = live ? min(t0 + per, h2) : t0;
      T* x = row + hh * HD;
      float ss = 0.f;
      for (int t = t0; t < t1; ++t) {
        const float a = to_f32(x[t]), b = to_f32(x[t + h2]);
        ss += a * a + b * b;
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      if (!live) continue;
      const float r = 1.f / sqrtf(ss / (float)HD + eps);
      const float* g = hh < H ? gq : gk;
      for (int t = t0; t < t1; ++t) {
        const float2 c = cs[t];
        const float a = to_f32(x[t]) * r * g[t], b = to_f32(x[t + h2]) * r * g[t + h2];
        x[t] = from_f32<T>(a * c.x - b * c.y);
        x[t + h2] = from_f32<T>(b * c.x + a * c.y);
      }
      if (part == 0) (hh < H ? rq : rk)[i * H + (hh < H ? hh : hh - H)] = r;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < D / EV; c += blockDim.x) {
      reinterpret_cast<uint4*>(qout + i * ldq)[c] = reinterpret_cast<const uint4*>(row)[c];
      reinterpret_cast<uint4*>(kring + slot * ldkv)[c] = reinterpret_cast<const uint4*>(row + D)[c];
    }
    __syncthreads();
  }
}

// QK-norm + RoPE forward without shared memory: a group of 8 lanes per q or
// k head (4 heads per warp, warps walk (token, head group) tasks); lane l of a
// group holds the 16-byte vectors l, l + 8 of both halves of the head
// (elements t and t + hd/2 are rotated together), the head's sum of squares
// is reduced over the group with shuffles, and the rotated halves go straight
// to q or the key ring.  Every access is a 16-byte vector and no block-wide
// barrier separates the loads of one token from the stores of another.
// Needs (hd/2) a multiple of 16 bytes of elements and at most 16 vectors per
// half (head_dim <= 128 in bf16, <= 64 in fp32 - larger heads take the
// kernel above).  The v rows are copied to the value ring by the same grid.
template <typename T>
__global__ void __launch_bounds__(256) qknorm_rope_fwd_warp_kernel(
    const T* __restrict__ qkv, int64_t ldqkv, const float* __restrict__ gq, const float* __restrict__ gk, int64_t n,
    int64_t p0, int H, int HD, float eps, const float2* __restrict__ tab, int64_t tab_p0, T* __restrict__ qout,
    int64_t ldq, T* __restrict__ kring, T* __restrict__ vring, int64_t ldkv, int64_t R, float* __restrict__ rq,
    float* __restrict__ rk) {
  constexpr int EV = 16 / sizeof(T);
  const int lane = threadIdx.x & 31, sub = lane & 7, hw = lane >> 3;
  const int h2 = HD / 2, NV = h2 / EV;
  const int hg = (2 * H + 3) / 4;  // groups of 4 among the 2H q and k heads
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < n * hg; w += nwarps) {
    const int64_t i = w / hg;
    const int hh = (int)(w % hg) * 4 + hw;  // q head hh < H, else k head hh - H
    const bool live = hh < 2 * H;
    const T* x = qkv + i * ldqkv + (int64_t)hh * HD;
    uint4 va[2], vb[2];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int v = sub + 8 * u;
      if (live && v < NV) {
        va[u] = *reinterpret_cast<const uint4*>(x + v * EV);
        vb[u] = *reinterpret_cast<const uint4*>(x + h2 + v * EV);
        const T* ea = reinterpret_cast<const T*>(&va[u]);
        const T* eb = reinterpret_cast<const T*>(&vb[u]);
#pragma unroll
        for (int e = 0; e < EV; ++e) {
          const float fa = to_f32(ea[e]), fb = to_f32(eb[e]);
          ss = fmaf(fa, fa, fmaf(fb, fb, ss));
        }
      }
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    if (!live) continue;
    const float r = 1.f / sqrtf(ss / (float)HD + eps);
    const bool is_q = hh < H;
    const float* g = is_q ? gq : gk;
    const float2* cs = tab + (p0 + i - tab_p0) * h2;
    T* dst = is_q ? qout + i * ldq + (int64_t)hh * HD : kring + ((p0 + i) % R) * ldkv + (int64_t)(hh - H) * HD;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int v = sub + 8 * u;
      if (v < NV) {
        const T* ea = reinterpret_cast<const T*>(&va[u]);
        const T* eb = reinterpret_cast<const T*>(&vb[u]);
        // the vector's gains and (cos, sin) pairs as 16-byte loads
        float ga[EV], gb[EV], cc[2 * EV];
#pragma unroll
        for (int e = 0; e < EV; e += 4) {
          *reinterpret_cast<float4*>(ga + e) = *reinterpret_cast<const float4*>(g + v * EV + e);
          *reinterpret_cast<float4*>(gb + e) = *reinterpret_cast<const float4*>(g + h2 + v * EV + e);
        }
#pragma unroll
        for (int e = 0; e < 2 * EV; e += 4)
          *reinterpret_cast<float4*>(cc + e) = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(cs + v * EV) + e);
        uint4 oa, ob;
        T* pa = reinterpret_cast<T*>(&oa);
        T* pb = reinterpret_cast<T*>(&ob);
#pragma unroll
        for (int e = 0; e < EV; ++e) {
          const float a = to_f32(ea[e]) * r * ga[e], b = to_f32(eb[e]) * r * gb[e];
          const float cx = cc[2 * e], sy = cc[2 * e + 1];
          pa[e] = from_f32<T>(a * cx - b * sy);
          pb[e] = from_f32<T>(b * cx + a * sy);
        }
        *reinterpret_cast<uint4*>(dst + v * EV) = oa;
        *reinterpret_cast<uint4*>(dst + h2 + v * EV) = ob;
      }
    }
    if (sub == 0) (is_q ? rq : rk)[i * H + (is_q ? hh : hh - H)] = r;
  }
  // v rows into the value ring
  const int64_t D = (int64_t)H * HD, dv = D / EV;
  const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n * dv; k += nthreads) {
    const int64_t i = k / dv, c = k % dv;
    reinterpret_cast<uint4*>(vring + ((p0 + i) % R) * ldkv)[c] =
        reinterpret_cast<const uint4*>(qkv + i * ldqkv + 2 * D)[c];
  }
}

// Backward of QK-norm + RoPE, in place on the q and k parts of dqkv, with the
// same staging as the forward: the token's dq|dk and raw q|k rows in smem,
// four threads per head.
template <typename T>
__global__ void __launch_bounds__(ROPE_THREADS) qknorm_rope_bwd_kernel(
    T* __restrict__ dqkv, int64_t ld, const T* __restrict__ qkv, int64_t ldqkv, const float* __restrict__ gq,
    const float* __restrict__ gk, const float* __restrict__ rq, const float* __restrict__ rk, int64_t n, int64_t p0,
    int H, int HD, const float2* __restrict__ tab, int64_t tab_p0) {
  extern __shared__ __align__(16) unsigned char rope_smem[];
  const int D = H * HD, h2 = HD / 2;
  T* drow = reinterpret_cast<T*>(rope_smem);  // [2 * D]: dq | dk
  T* xrow = drow + 2 * D;                     // [2 * D]: raw q | k
  constexpr int EV = 16 / sizeof(T);
  const int per = (h2 + 3) / 4;
  const int tasks = ((8 * H + 31) / 32) * 32;
  for (int64_t i = blockIdx.x; i < n; i += gridDim.x) {
    for (int c = threadIdx.x; c < 2 * D / EV; c += blockDim.x) {
      reinterpret_cast<uint4*>(drow)[c] = reinterpret_cast<const uint4*>(dqkv + i * ld)[c];
      reinterpret_cast<uint4*>(xrow)[c] = reinterpret_cast<const uint4*>(qkv + i * ldqkv)[c];
    }
    __syncthreads();
    const float2* cs = tab + (p0 + i - tab_p0) * h2;
    for (int task = threadIdx.x; task < tasks; task += blockDim.x) {
      const int hh = task / 4, part = task % 4;
      const bool live = hh < 2 * H;
      const int t0 = part * per, t1 = live ? min(t0 + per, h2) : t0;
      const int h = hh < H ? hh : hh - H;
      const float* g = hh < H ? gq : gk;
      const float r = live ? (hh < H ? rq : rk)[i * H + h] : 0.f;
      T* dv = drow + hh * HD;
      const T* xv = xrow + hh * HD;
      float dot = 0.f;
      for (int t = t0; t < t1; ++t) {
        const float2 c = cs[t];
        const float d1 = to_f32(dv[t]), d2 = to_f32(dv[t + h2]);
        // transpose of the rotation, then the gain
        const float u1 = (d1 * c.x + d2 * c.y) * g[t], u2 = (d2 * c.x - d1 * c.y) * g[t + h2];
        dot += to_f32(xv[t]) * r * u1 + to_f32(xv[t + h2]) * r * u2;
      }
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      dot += __shfl_xor_sync(0xffffffffu, dot, 2);
      if (!live) continue;
      const float dm = dot / (float)HD;
      for (int t = t0; t < t1; ++t) {
        const float2 c = cs[t];
        const float d1 = to_f32(dv[t]), d2 = to_f32(dv[t + h2]);
        const float u1 = (d1 * c.x + d2 * c.y) * g[t], u2 = (d2 * c.x - d1 * c.y) * g[t + h2];
        dv[t] = from_f32<T>(r * (u1 - to_f32(xv[t]) * r * dm));
        dv[t + h2] = from_f32<T>(r * (u2 - to_f32(xv[t + h2]) * r * dm));
      }
    }
    __syncthreads();
    for (int c = threadIdx.x; c < 2 * D / EV; c += blockDim.x)
      reinterpret_cast<uint4*>(dqkv + i * ld)[c] = reinterpret_cast<const uint4*>(drow)[c];
    __syncthreads();
  }
}

template <typename T>
__global__ void swiglu_bwd_kernel(const T* da, int64_t ldda, const T* gu, int64_t ldgu, int64_t n, int64_t nfeat,
                                  T* dgu, int64_t lddgu) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = blockIdx.y;
  if (j >= nfeat || row >= n) return;
  const int64_t gc = 128 * (j / 64) + (j % 64), uc = gc + 64;
  const float g = to_f32(gu[row * ldgu + gc]), u = to_f32(gu[row * ldgu + uc]);
  const float a = to_f32(da[row * ldda + j]);
  const float sg = 1.f / (1.f + expf(-g));
  dgu[row * lddgu + gc] = from_f32<T>(a * u * sg * (1.f + g * (1.f - sg)));
  dgu[row * lddgu + uc] = from_f32<T>(a * g * sg);
}

// Four consecutive features per thread (one 8- or 16-byte access per operand).
template <typename T> struct Vec4;
template <> struct Vec4<float> { using type = float4; };
template <> struct Vec4<bf16> { using type = uint2; };
__device__ __forceinline__ void unpack4(float4 v, float (&f)[4]) { f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w; }
__device__ __forceinline__ void unpack4(uint2 v, float (&f)[4]) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v.y));
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}
template <typename V> __device__ __forceinline__ V pack4(const float (&f)[4]);
template <> __device__ __forceinline__ float4 pack4<float4>(const float (&f)[4]) { return make_float4(f[0], f[1], f[2], f[3]); }
template <> __device__ __forceinline__ uint2 pack4<uint2>(const float (&f)[4]) {
  __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]), b = __floats2bfloat162_rn(f[2], f[3]);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  return u;
}

template <typename T>
__global__ void swiglu_bwd_vec_kernel(const T* da, int64_t ldda, const T* gu, int64_t ldgu, int64_t n, int64_t nfeat,
                                      T* dgu, int64_t lddgu) {
  using V = typename Vec4<T>::type;
  const int64_t j = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  const int64_t row = blockIdx.y;
  if (j >= nfeat || row >= n) return;
  const int64_t gc = 128 * (j / 64) + (j % 64), uc = gc + 64;
  float g[4], u[4], a[4], dg[4], du[4];
  unpack4(*reinterpret_cast<const V*>(gu + row * ldgu + gc), g);
  unpack4(*reinterpret_cast<const V*>(gu + row * ldgu + uc), u);
  unpack4(*reinterpret_cast<const V*>(da + row * ldda + j), a);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float sg = 1.f / (1.f + expf(-g[e]));
    dg[e] = a[e] * u[e] * sg * (1.f + g[e] * (1.f - sg));
    du[e] = a[e] * g[e] * sg;
  }
  *reinterpret_cast<V*>(dgu + row * lddgu + gc) = pack4<V>(dg);
  *reinterpret_cast<V*>(dgu + row * lddgu + uc) = pack4<V>(du);
}

// Combines the per-tile softmax partials of each row: a block covers 32 rows
// (threadIdx.x) and splits the tiles over CE_SLICES slices (threadIdx.y),
// each slice keeping an online (max, sum) pair, merged through smem.
constexpr int CE_SLICES = 16;

__global__ void __launch_bounds__(32 * CE_SLICES) ce_finalize_kernel(const float* pmax, const float* psum,
                                                                     int64_t part_ld, int tiles, const float* zt,
                                                                     int64_t n, int64_t n_valid, float inv_nc,
                                                                     float* loss_out, float* lse_out, float* scale) {
  __shared__ float sm_m[CE_SLICES][32], sm_s[CE_SLICES][32];
  const int64_t i = (int64_t)blockIdx.x * 32 + threadIdx.x;
  float M = -INFINITY, S = 0.f;
  if (i < n) {
#pragma unroll 4
    for (int t = threadIdx.y; t < tiles; t += CE_SLICES) {
      const float m = pmax[(int64_t)t * part_ld + i], ps = psum[(int64_t)t * part_ld + i];
      if (m == -INFINITY) continue;
      if (m > M) {
        S = S * expf(M - m) + ps;
        M = m;
      } else {
        S += ps * expf(m - M);
      }
    }
  }
  sm_m[threadIdx.y][threadIdx.x] = M;
  sm_s[threadIdx.y][threadIdx.x] = S;
  __syncthreads();
  if (threadIdx.y != 0 || i >= n) return;
  float Mt = -INFINITY;
  for (int y = 0; y < CE_SLICES; ++y) Mt = fmaxf(Mt, sm_m[y][threadIdx.x]);
  float St = 0.f;
  for (int y = 0; y < CE_SLICES; ++y) {
    const float m = sm_m[y][threadIdx.x];
    if (m > -INFINITY) St += sm_s[y][threadIdx.x] * expf(m - Mt);
  }
  const float lse = Mt + logf(St);
  lse_out[i] = lse;
  const bool ok = i < n_valid;
  loss_out[i] = ok ? lse - zt[i] : __int_as_float(0x7fc00000);
  scale[i] = ok ? inv_nc : 0.f;
}

// One thread per 8 columns of a row: two float4 loads of the logits and one
// 16-byte store of the bf16 gradient when the row segment is whole and
// aligned (the vocab chunks used here always are); element by element at a
// ragged end.
template <typename T>
__global__ void ce_grad_kernel(const float* z, int64_t ldz, const float* lse, const float* scale, const int32_t* tgt,
                               int64_t col0, int64_t n, int64_t ncols, T* dz, int64_t lddz) {
  constexpr float LOG2E = 1.4426950408889634f;
  const int64_t g8 = (ncols + 7) / 8;
  const int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gi >= n * g8) return;
  const int64_t row = gi / g8, c = (gi % g8) * 8;
  const float l = lse[row], sc = scale[row];
  const int64_t t = (int64_t)tgt[row] - col0;
  const float* zr = z + row * ldz + col0 + c;
  T* out = dz + row * lddz + c;
  const int cnt = (int)(ncols - c < 8 ? ncols - c : 8);
  const bool vec = cnt == 8 && (reinterpret_cast<uintptr_t>(zr) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(out) & 15) == 0 && sizeof(T) == 2;
  float v[8];
  if (vec) {
    const float4 x0 = *reinterpret_cast<const float4*>(zr), x1 = *reinterpret_cast<const float4*>(zr + 4);
    v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
    v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
  } else {
    for (int e = 0; e < 8; ++e) v[e] = e < cnt ? zr[e] : 0.f;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = (exp2f((v[e] - l) * LOG2E) - (c + e == t ? 1.f : 0.f)) * sc;
  if (vec) {
    uint4 w;
    T* pw = reinterpret_cast<T*>(&w);
#pragma unroll
    for (int e = 0; e < 8; ++e) pw[e] = from_f32<T>(v[e]);
    *reinterpret_cast<uint4*>(out) = w;
  } else {
    for (int e = 0; e < cnt; ++e) out[e] = from_f32<T>(v[e]);
  }
}

__global__ void check_tokens_kernel(const int32_t* tok, int64_t T, int V, int* err) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T) return;
  const int32_t t = tok[i];
  if (t < 0 || t >= V) atomicOr(err, DEV_ERR_BAD_TOKEN);
}

__global__ void chunk_targets_kernel(const int32_t* tok, int64_t T, int64_t p0, int64_t n, int32_t* targets) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  targets[i] = (p0 + i + 1 < T) ? tok[p0 + i + 1] : -1;
}

template <typename TS, typename TD>
__global__ void interleave_kernel(const TS* gate, const TS* up, int f, int d, TD* out) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)2 * f * d) return;
  const int64_t r = idx / d, c = idx % d;
  const int64_t pair = r / 128, l = r % 128;
  const TS v = l < 64 ? gate[(64 * pair + l) * d + c] : up[(64 * pair + l - 64) * d + c];
  out[idx] = from_f32<TD>(to_f32(v));
}

__global__ void deinterleave_kernel(const float* in, int f, int d, float* gate, float* up) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)2 * f * d) return;
  const int64_t r = idx / d, c = idx % d;
  const int64_t pair = r / 128, l = r % 128;
  if (l < 64) gate[(64 * pair + l) * d + c] = in[idx];
  else up[(64 * pair + l - 64) * d + c] = in[idx];
}

template <typename TS, typename TD>
__global__ void copy2d_kernel(const TS* src, int64_t lds, TD* dst, int64_t ldd, int64_t rows, int64_t cols) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * cols) return;
  const int64_t r = idx / cols, c = idx % cols;
  dst[r * ldd + c] = from_f32<TD>(to_f32(src[r * lds + c]));
}

// lo = bf16(x - bf16(x)): the low half of a two-term bf16 representation of x
__global__ void bf16_lo_kernel(const float* src, int64_t lds, bf16* dst, int64_t ldd, int64_t rows, int64_t cols) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * cols) return;
  const int64_t r = idx / cols, c = idx % cols;
  const float x = src[r * lds + c];
  dst[r * ldd + c] = __float2bfloat16_rn(x - __bfloat162float(__float2bfloat16_rn(x)));
}

inline unsigned row_blocks(int64_t rows) { return ceil_div(rows, ROW_WARPS); }

}  // namespace

template <typename T>
int embed_gather(const int32_t* tok, const T* E, int64_t n, int d, int V, float* x, int* err, cudaStream_t s) {
  embed_kernel<T><<<row_blocks(n), 32 * ROW_WARPS, 0, s>>>(tok, E, n, d, V, x, err);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <typename T>
int rmsnorm_fwd(const float* x, int64_t ldx, const float* g, float eps, int64_t n, int d, T* y, int64_t ldy,
                float* rstd, cudaStream_t s) {
  if (n <= 0) return TTT_OK;
  if (d % 4 == 0 && d <= 4 * VT * VN && ldx % 4 == 0 && ldy % 4 == 0 && al(x, 16) && al(g, 16) && al(y, 4 * sizeof(T)))
    rmsnorm_fwd_vec_kernel<T><<<(unsigned)n, VT, 0, s>>>(x, ldx, g, eps, d, y, ldy, rstd);
  else
    rmsnorm_fwd_kernel<T><<<row_blocks(n), 32 * ROW_WARPS, 0, s>>>(x, ldx, g, eps, n, d, y, ldy, rstd);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <typename T>
int rmsnorm_bwd(const float* x, int64_t ldx, const float* rstd, const float* g, const float* dy, int64_t lddy,
                const float* dres, int64_t ldres, int64_t n, int d, float* dx, int64_t lddx, T* dx16, int64_t ld16,
                cudaStream_t s) {
  if (n <= 0) return TTT_OK;
  if (d % 4 == 0 && d <= 4 * VT * VN && ldx % 4 == 0 && lddy % 4 == 0 && lddx % 4 == 0 && (!dres || ldres % 4 == 0) &&
      (!dx16 || ld16 % 4 == 0) && al(x, 16) && al(g, 16) && al(dy, 16) && al(dres, 16) && al(dx, 16) &&
      al(dx16, 4 * sizeof(T)))
    rmsnorm_bwd_vec_kernel<T><<<(unsigned)n, VT, 0, s>>>(x, ldx, rstd, g, dy, lddy, dres, ldres, d, dx, lddx, dx16,
                                                         ld16);
  else
    rmsnorm_bwd_kernel<T><<<row_blocks(n), 32 * ROW_WARPS, 0, s>>>(x, ldx, rstd, g, dy, lddy, dres, ldres, n, d, dx,
                                                                    lddx, dx16, ld16);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <typename T>
int qknorm_rope_fwd(const T* qkv, int64_t ldqkv, const float* gq, const float* gk, int64_t n, int64_t p0, int H,
                    int HD, float eps, const float2* tab, int64_t tab_p0, T* qout, int64_t ldq, T* kring, T* vring,
                    int64_t ldkv, int64_t R, float* rq, float* rk, cudaStream_t s) {
  if (HD % 2) return set_error(TTT_ERR_UNSUPPORTED, "qknorm_rope: odd head_dim");
  if (n <= 0) return TTT_OK;
  constexpr int EV = 16 / (int)sizeof(T);
  const int64_t D = (int64_t)H * HD;
  const bool vec_ok = D % EV == 0 && ldqkv % EV == 0 && ldq % EV == 0 && ldkv % EV == 0 &&
                      reinterpret_cast<uintptr_t>(qkv) % 16 == 0 && reinterpret_cast<uintptr_t>(qout) % 16 == 0 &&
                      reinterpret_cast<uintptr_t>(kring) % 16 == 0 && reinterpret_cast<uintptr_t>(vring) % 16 == 0;
  if (!vec_ok) return set_error(TTT_ERR_INVALID_ARG, "qknorm_rope: rows must be 16-byte aligned");
  const bool al = reinterpret_cast<uintptr_t>(gq) % 16 == 0 && reinterpret_cast<uintptr_t>(gk) % 16 == 0 &&
                  reinterpret_cast<uintptr_t>(tab) % 16 == 0 && (HD / 2) % 4 == 0;
  if (al && (HD / 2) % EV == 0 && (HD / 2) / EV <= 16) {
    const int64_t tasks = n * ((2 * H + 3) / 4);  // warps of work
    const unsigned grid = (unsigned)std::min<int64_t>((tasks + 7) / 8, 148 * 16);
    qknorm_rope_fwd_warp_kernel<T><<<grid, 256, 0, s>>>(qkv, ldqkv, gq, gk, n, p0, H, HD, eps, tab, tab_p0, qout, ldq,
                                                        kring, vring, ldkv, R, rq, rk);
    TTT_CUDA_TRY(cudaGetLastError());
    return TTT_OK;
  }
  const size_t smem = 2 * (size_t)D * sizeof(T);
  if (smem > 48 * 1024) return set_error(TTT_ERR_UNSUPPORTED, "qknorm_rope: q and k rows exceed 48 KB");
  const unsigned grid = (unsigned)std::min<int64_t>(n, 148 * 8);
  qknorm_rope_fwd_kernel<T><<<grid, ROPE_THREADS, smem, s>>>(qkv, ldqkv, gq, gk, n, p0, H, HD, eps, tab, tab_p0,
                                                             qout, ldq, kring, vring, ldkv, R, rq, rk);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <typename T>
int qknorm_rope_bwd(T* dqkv, int64_t ld, const T* qkv, int64_t ldqkv, const float* gq, const float* gk,
                    const float* rq, const float* rk, int64_t n, int64_t p0, int H, int HD, const float2* tab,
                    int64_t tab_p0, cudaStream_t s) {
  if (HD % 2) return set_error(TTT_ERR_UNSUPPORTED, "qknorm_rope: odd head_dim");
  if (n <= 0) return TTT_OK;
  constexpr int EV = 16 / (int)sizeof(T);
  const int64_t D = (int64_t)H * HD;
  if (D % EV || ld % EV || ldqkv % EV || reinterpret_cast<uintptr_t>(dqkv) % 16 || reinterpret_cast<uintptr_t>(qkv) % 16)
    return set_error(TTT_ERR_INVALID_ARG, "qknorm_rope_bwd: rows must be 16-byte aligned");
  const size_t smem = 4 * (size_t)D * sizeof(T);
  if (smem > 48 * 1024) return set_error(TTT_ERR_UNSUPPORTED, "qknorm_rope_bwd: rows exceed 48 KB of smem");
  const unsigned grid = (unsigned)std::min<int64_t>(n, 148 * 8);
  qknorm_rope_bwd_kernel<T><<<grid, ROPE_THREADS, smem, s>>>(dqkv, ld, qkv, ldqkv, gq, gk, rq, rk, n, p0, H, HD, tab,
                                                             tab_p0);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <typename T>
int swiglu_bwd(const T* da, int64_t ldda, const T* gu, int64_t ldgu, int64_t n, int64_t nfeat, T* dgu,
               int64_t lddgu, cudaStream_t s) {
  if (nfeat % 64) return set_error(TTT_ERR_INVALID_ARG, "swiglu_bwd: features must be a multiple of 64");
  dim3 grid(ceil_div(nfeat, 256), (unsigned)n);
  constexpr int VB = 4 * (int)sizeof(T);  // bytes of a 4-feature access
  const bool vec = ldda % 4 == 0 && ldgu % 4 == 0 && lddgu % 4 == 0 && reinterpret_cast<uintptr_t>(da) % VB == 0 &&
                   reinterpret_cast<uintptr_t>(gu) % VB == 0 && reinterpret_cast<uintptr_t>(dgu) % VB == 0;
  if (vec) {
    dim3 g4(ceil_div(nfeat / 4, 256), (unsigned)n);
    swiglu_bwd_vec_kernel<T><<<g4, 256, 0, s>>>(da, ldda, gu, ldgu, n, nfeat, dgu, lddgu);
  } else {
    swiglu_bwd_kernel<T><<<grid, 256, 0, s>>>(da, ldda, gu, ldgu, n, nfeat, dgu, lddgu);
  }
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

int ce_finalize(const float* pmax, const float* psum, int64_t part_ld, int tiles, const float* zt, int64_t n,
                int64_t n_valid, float inv_nc, float* loss_out, float* lse, float* scale, cudaStream_t s) {
  if (n <= 0) return TTT_OK;
  ce_finalize_kernel<<<ceil_div(n, 32), dim3(32, CE_SLICES), 0, s>>>(pmax, psum, part_ld, tiles, zt, n, n_valid,
                                                                     inv_nc, loss_out, lse, scale);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <typename T>
int ce_grad_from_logits(const float* z, int64_t ldz, const float* lse, const float* scale, const int32_t* tgt,
                        int64_t col0, int64_t n, int64_t ncols, T* dz, int64_t lddz, cudaStream_t s) {
  if (n <= 0 || ncols <= 0) return TTT_OK;
  ce_grad_kernel<T><<<ceil_div(n * ((ncols + 7) / 8), 256), 256, 0, s>>>(z, ldz, lse, scale, tgt, col0, n, ncols, dz,
                                                                          lddz);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}
template int ce_grad_from_logits<float>(const float*, int64_t, const float*, const float*, const int32_t*, int64_t,
                                        int64_t, int64_t, float*, int64_t, cudaStream_t);
template int ce_grad_from_logits<bf16>(const float*, int64_t, const float*, const float*, const int32_t*, int64_t,
                                       int64_t, int64_t, bf16*, int64_t, cudaStream_t);

int check_tokens(const int32_t* tok, int64_t T, int V, int* err, cudaStream_t s) {
  check_tokens_kernel<<<ceil_div(T, 256), 256, 0, s>>>(tok, T, V, err);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

int chunk_targets(const int32_t* tok, int64_t T, int64_t p0, int64_t n, int32_t* targets, cudaStream_t s) {
  chunk_targets_kernel<<<ceil_div(n, 256), 256, 0, s>>>(tok, T, p0, n, targets);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <typename TS, typename TD>
int interleave_gate_up(const TS* gate, const TS* up, int f, int d, TD* out, cudaStream_t s) {
  if (f % 64) return set_error(TTT_ERR_INVALID_ARG, "interleave: d_ff must be a multiple of 64");
  interleave_kernel<TS, TD><<<ceil_div((int64_t)2 * f * d, 256), 256, 0, s>>>(gate, up, f, d, out);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}
template int interleave_gate_up<float, float>(const float*, const float*, int, int, float*, cudaStream_t);
template int interleave_gate_up<bf16, bf16>(const bf16*, const bf16*, int, int, bf16*, cudaStream_t);

int deinterleave_gate_up(const float* in, int f, int d, float* gate, float* up, cudaStream_t s) {
  deinterleave_kernel<<<ceil_div((int64_t)2 * f * d, 256), 256, 0, s>>>(in, f, d, gate, up);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <typename T>
int copy2d_from_f32(const float* src, int64_t lds, T* dst, int64_t ldd, int64_t rows, int64_t cols, cudaStream_t s) {
  copy2d_kernel<float, T><<<ceil_div(rows * cols, 256), 256, 0, s>>>(src, lds, dst, ldd, rows, cols);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

int rope_table(float2* tab, int64_t p0, int64_t n, int HD, double theta, cudaStream_t s) {
  if (n <= 0) return TTT_OK;
  if (HD % 2) return set_error(TTT_ERR_UNSUPPORTED, "rope_table: odd head_dim");
  rope_table_kernel<<<ceil_div(n * (HD / 2), 256), 256, 0, s>>>(tab, p0, n, HD, theta);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

int bf16_lo2d(const float* src, int64_t lds, bf16* dst, int64_t ldd, int64_t rows, int64_t cols, cudaStream_t s) {
  if (rows * cols == 0) return TTT_OK;
  bf16_lo_kernel<<<ceil_div(rows * cols, 256), 256, 0, s>>>(src, lds, dst, ldd, rows, cols);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <typename T>
int copy2d(const T* src, int64_t lds, T* dst, int64_t ldd, int64_t rows, int64_t cols, cudaStream_t s) {
  copy2d_kernel<T, T><<<ceil_div(rows * cols, 256), 256, 0, s>>>(src, lds, dst, ldd, rows, cols);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

#define TTT_INST(T)                                                                                              \
  template int embed_gather<T>(const int32_t*, const T*, int64_t, int, int, float*, int*, cudaStream_t);        \
  template int rmsnorm_fwd<T>(const float*, int64_t, const float*, float, int64_t, int, T*, int64_t, float*,    \
                              cudaStream_t);                                                                    \
  template int rmsnorm_bwd<T>(const float*, int64_t, const float*, const float*, const float*, int64_t,         \
                              const float*, int64_t, int64_t, int, float*, int64_t, T*, int64_t, cudaStream_t); \
  template int qknorm_rope_fwd<T>(const T*, int64_t, const float*, const float*, int64_t, int64_t, int, int,    \
                                  float, const float2*, int64_t, T*, int64_t, T*, T*, int64_t, int64_t, float*, \
                                  float*, cudaStream_t);                                                        \
  template int qknorm_rope_bwd<T>(T*, int64_t, const T*, int64_t, const float*, const float*, const float*,     \
                                  const float*, int64_t, int64_t, int, int, const float2*, int64_t,             \
                                  cudaStream_t);                                                                \
  template int swiglu_bwd<T>(const T*, int64_t, const T*, int64_t, int64_t, int64_t, T*, int64_t, cudaStream_t); \
  template int copy2d_from_f32<T>(const float*, int64_t, T*, int64_t, int64_t, int64_t, cudaStream_t);          \
  template int copy2d<T>(const T*, int64_t, T*, int64_t, int64_t, int64_t, cudaStream_t);

TTT_INST(float)
TTT_INST(bf16)

}  // namespace ttt
