// Tensor-core GEMM for sm_100a: TMA tile loads into 128B-swizzled shared
// memory, tcgen05.mma (kind::f16, bf16 x bf16 -> fp32) issued by one thread,
// accumulator in TMEM, and a fused epilogue read back with tcgen05.ld.
//
// CTA = 6 warps: warp 0 lane 0 issues TMA, warp 1 owns the TMEM allocation
// and lane 0 issues the MMAs, warps 2..5 run the epilogue (warp w reads TMEM
// lanes 32*(w%4) .. +31, one accumulator row per thread).  Tile 128 x BN x 64,
// BN in {128, 256}, a 4- or 6-stage smem ring between producer and MMA.
#include <algorithm>
#include <map>
#include <mutex>
#include <set>

#include "gemm.cuh"
#include "ptx.cuh"

namespace ttt {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;

// Warps: 0 = TMA producer, 1 = MMA issuer, 2 .. 9 = two epilogue groups of four
// (one per TMEM accumulator buffer, so two units drain at the same time).
constexpr int kEpiWarps = 8;
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;

// Row pitch (floats) of an epilogue warp's 32 x 32 transpose tile: 33 for the
// scalar column-per-lane reads, 36 for the SGD epilogue's float4 reads (rows
// then start on 16-byte boundaries, and both the float4 writes of a row and
// the float4 reads of four rows by eight lanes each hit 32 distinct banks).
template <int EPI>
constexpr int kWStride = EPI == EPI_SGD ? 36 : 33;

template <int BN, int EPI>
struct TcCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  // the SGD GEMMs reduce over one chunk (K = b): one stage fewer pays for the wider transpose tiles
  static constexpr int STAGES = ((BN == 256) ? 4 : 6) - (EPI == EPI_SGD ? 1 : 0);
  static constexpr int WBUF = kEpiWarps * 32 * kWStride<EPI> * 4;  // epilogue transpose tiles, one per epilogue warp
  static constexpr int SMEM = STAGES * STAGE + 1024 /*align*/ + 256 /*barriers*/ + WBUF;
  static_assert(SMEM <= 232448, "shared memory per block");
};

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.f + __expf(-g)) * u; }

template <typename T>
__device__ __forceinline__ void store32(T* dst, const float* v, int nvalid);

template <>
__device__ __forceinline__ void store32<float>(float* dst, const float* v, int nvalid) {
  if (nvalid >= 32 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
  } else {
    for (int i = 0; i < nvalid && i < 32; ++i) dst[i] = v[i];
  }
}

template <>
__device__ __forceinline__ void store32<bf16>(bf16* dst, const float* v, int nvalid) {
  if (nvalid >= 32 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
      uint4 w;
      __nv_bfloat162 p0 = __floats2bfloat162_rn(v[i], v[i + 1]);
      __nv_bfloat162 p1 = __floats2bfloat162_rn(v[i + 2], v[i + 3]);
      __nv_bfloat162 p2 = __floats2bfloat162_rn(v[i + 4], v[i + 5]);
      __nv_bfloat162 p3 = __floats2bfloat162_rn(v[i + 6], v[i + 7]);
      w.x = *reinterpret_cast<uint32_t*>(&p0);
      w.y = *reinterpret_cast<uint32_t*>(&p1);
      w.z = *reinterpret_cast<uint32_t*>(&p2);
      w.w = *reinterpret_cast<uint32_t*>(&p3);
      *reinterpret_cast<uint4*>(dst + i) = w;
    }
  } else {
    for (int i = 0; i < nvalid && i < 32; ++i) dst[i] = __float2bfloat16_rn(v[i]);
  }
}

__device__ __forceinline__ void ld32f(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  __syncwarp();
  ptx::tmem_ld32(taddr, r);
  ptx::tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Epilogue of one accumulator row (thread) over the tile's BN columns.
template <int BN, int EPI, typename TACT>
__device__ __forceinline__ void epilogue_row(uint32_t t_row, int64_t row, bool row_ok, int64_t n0, int64_t N,
                                             const EpiArgs& ep, int tile_n, int split) {
  float v[32];
  if constexpr (EPI == EPI_SWIGLU) {
#pragma unroll 1
    for (int j = 0; j < BN / 128; ++j) {
#pragma unroll 1
      for (int h = 0; h < 64; h += 32) {
        float u[32];
        ld32f(t_row + 128 * j + h, v);
        ld32f(t_row + 128 * j + 64 + h, u);
        const int64_t gcol = n0 + 128 * j + h;
        if (!row_ok || gcol >= N) continue;
        if (ep.c2) {
          TACT* raw = reinterpret_cast<TACT*>(ep.c2) + row * ep.ldc2 + gcol;
          store32<TACT>(raw, v, 32);
          store32<TACT>(raw + 64, u, 32);
        }
        float a[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = silu_mul(v[i], u[i]);
        TACT* out = reinterpret_cast<TACT*>(ep.c) + row * ep.ldc + (n0 / 2 + 64 * j + h);
        store32<TACT>(out, a, 32);
      }
    }
  } else if constexpr (EPI == EPI_CE_FWD) {
    constexpr float LOG2E = 1.4426950408889634f;
    float mx = -INFINITY, sm = 0.f, zt = 0.f;
    bool found = false;
    const int64_t tgt = row_ok ? (int64_t)ep.row_i[row] - ep.col_offset : -1;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      ld32f(t_row + c, v);
      const int64_t col0 = n0 + c;
      const int nval = (int)(N - col0 < 32 ? N - col0 : 32);
      if (ep.c && row_ok && nval > 0)  // keep the logits for the backward (instead of recomputing them)
        store32<float>(reinterpret_cast<float*>(ep.c) + row * ep.ldc + col0, v, nval);
      float cm = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < nval) cm = fmaxf(cm, v[i]);
      if (nval <= 0) continue;
      if (cm > mx) {
        sm *= exp2f((mx - cm) * LOG2E);
        mx = cm;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < nval) sm += exp2f((v[i] - mx) * LOG2E);
      if (tgt >= col0 && tgt < col0 + nval) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (col0 + i == tgt) zt = v[i];
        found = true;
      }
    }
    if (row_ok) {
      ep.part_max[(int64_t)tile_n * ep.part_ld + row] = mx;
      ep.part_sum[(int64_t)tile_n * ep.part_ld + row] = sm;
      if (found) ep.target_logit[row] = zt;
    }
  } else {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      ld32f(t_row + c, v);
      const int64_t col0 = n0 + c;
      if (!row_ok || col0 >= N) continue;
      const int nval = (int)(N - col0 < 32 ? N - col0 : 32);
      if constexpr (EPI == EPI_STORE_BF16) {
        store32<bf16>(reinterpret_cast<bf16*>(ep.c) + row * ep.ldc + col0, v, nval);
      } else if constexpr (EPI == EPI_CE_BWD) {
        constexpr float LOG2E = 1.4426950408889634f;
        const float lse = ep.row_f[row], sc = ep.row_g[row];
        const int64_t tgt = (int64_t)ep.row_i[row] - ep.col_offset;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float p = exp2f((v[i] - lse) * LOG2E);
          v[i] = (p - (col0 + i == tgt ? 1.f : 0.f)) * sc;
        }
        store32<TACT>(reinterpret_cast<TACT*>(ep.c) + row * ep.ldc + col0, v, nval);
      }
    }
  }
}

// fp32 stores and read-modify-write epilogues (EPI_STORE_F32, EPI_ADD_F32,
// EPI_SGD) go through a per-warp transpose so that global accesses run along
// rows with lane = column (coalesced 128-byte lines).  The warp owns rows
// row0 .. row0+31 of the tile.  Its read source (the residual or the master)
// does not depend on the accumulator, so it is read ahead: two register
// buffers of one 32 x 32 chunk each alternate between the even and the odd
// chunks, the first two chunks are loaded before the accumulator is ready,
// and each row's value for the chunk two steps ahead is loaded as soon as
// that row's current value has been used.  Two chunks of loads (8 KB per
// warp) stay in flight through the whole tile, which the HBM-bound SGD
// epilogue needs to keep enough bytes in flight per SM.
template <int EPI>
constexpr bool kTransposedEpi = EPI == EPI_STORE_F32 || EPI == EPI_ADD_F32 || EPI == EPI_SGD;

template <int EPI>
constexpr bool kEpiReads = EPI == EPI_ADD_F32 || EPI == EPI_SGD;

// Read source of a read-modify-write epilogue and its leading dimension.
template <int EPI>
__device__ __forceinline__ const float* epi_src(const EpiArgs& ep, int64_t& ld) {
  ld = ep.ldc;
  if constexpr (EPI == EPI_ADD_F32) {
    if (ep.c2) {
      ld = ep.ldc2;
      return reinterpret_cast<const float*>(ep.c2);
    }
  }
  return reinterpret_cast<const float*>(ep.c);
}

template <int EPI>
__device__ __forceinline__ void epi_load_chunk(const EpiArgs& ep, int64_t row0, int64_t M, int64_t col, int64_t N,
                                               float (&dst)[32]) {
  if constexpr (kEpiReads<EPI>) {
    int64_t ld;
    const float* src = epi_src<EPI>(ep, ld);
    const int nrows = (int)(M - row0 < 32 ? M - row0 : 32);
    const float* p = src + row0 * ld + col;
    if (col < N && nrows == 32) {
#pragma unroll
      for (int r = 0; r < 32; ++r, p += ld) dst[r] = *p;
    } else {
      const bool col_ok = col < N;
#pragma unroll
      for (int r = 0; r < 32; ++r, p += ld) dst[r] = (col_ok && r < nrows) ? *p : 0.f;
    }
  }
}

// One 32 x 32 chunk (rows row0.., column col of this lane): writes it from the
// transposed accumulator in wbuf when `store`, with buf[r] as row r's read
// source; then, when `nsrc` is set (this lane's column two chunks ahead,
// already offset to row0), refills buf[r] from it right after its use.
template <int EPI, bool CHECK, bool HI, bool LO>
__device__ __forceinline__ void epi_chunk(const EpiArgs& ep, int64_t row0, int64_t col, int split, int nrows,
                                          bool store, const float* wbuf, float (&buf)[32], const float* nsrc,
                                          int64_t nld) {
  const int lane = threadIdx.x & 31;
  if constexpr (EPI == EPI_STORE_F32) {
    if (!store) return;
    float* p = reinterpret_cast<float*>(ep.c) + (int64_t)split * ep.split_stride + row0 * ep.ldc + col;
#pragma unroll
    for (int r = 0; r < 32; ++r, p += ep.ldc)
      if (!CHECK || r < nrows) *p = wbuf[r * 33 + lane];
  } else if constexpr (EPI == EPI_ADD_F32) {
    float* p = reinterpret_cast<float*>(ep.c) + row0 * ep.ldc + col;
#pragma unroll
    for (int r = 0; r < 32; ++r, p += ep.ldc) {
      if (store && (!CHECK || r < nrows)) *p = buf[r] + wbuf[r * 33 + lane];
      if (nsrc) buf[r] = (!CHECK || r < nrows) ? nsrc[r * nld] : 0.f;
    }
  } else {  // EPI_SGD
    float* p = reinterpret_cast<float*>(ep.c) + row0 * ep.ldc + col;
    bf16* ph = HI ? reinterpret_cast<bf16*>(ep.c2) + row0 * ep.ldc2 + col : nullptr;
    bf16* pl = LO ? reinterpret_cast<bf16*>(ep.c3) + row0 * ep.ldc3 + col : nullptr;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      if (store && (!CHECK || r < nrows)) {
        const float w = __fmaf_rn(-ep.alpha, wbuf[r * 33 + lane], buf[r]);
        *p = w;
        if constexpr (HI) {
          const bf16 hi = __float2bfloat16_rn(w);
          *ph = hi;
          if constexpr (LO) *pl = __float2bfloat16_rn(w - __bfloat162float(hi));
        }
      }
      if (nsrc) buf[r] = (!CHECK || r < nrows) ? nsrc[r * nld] : 0.f;
      p += ep.ldc;
      if constexpr (HI) ph += ep.ldc2;
      if constexpr (LO) pl += ep.ldc3;
    }
  }
}

template <int EPI, bool HI, bool LO>
__device__ __forceinline__ void epi_chunk_check(const EpiArgs& ep, int64_t row0, int64_t col, int split, int nrows,
                                                bool store, const float* wbuf, float (&buf)[32], const float* nsrc,
                                                int64_t nld) {
  if (nrows == 32)
    epi_chunk<EPI, false, HI, LO>(ep, row0, col, split, nrows, store, wbuf, buf, nsrc, nld);
  else
    epi_chunk<EPI, true, HI, LO>(ep, row0, col, split, nrows, store, wbuf, buf, nsrc, nld);
}

// bufA / bufB hold the read source of chunks 0 and 1 on entry.
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_transposed(uint32_t t_row, const EpiArgs& ep, int64_t n0, int64_t N,
                                                    int split, float* wbuf, int64_t row0, int64_t M,
                                                    float (&bufA)[32], float (&bufB)[32]) {
  static_assert(BN % 32 == 0, "32-column chunks");
  const int lane = threadIdx.x & 31;
  const int nrows = (int)(M - row0 < 32 ? (M - row0 > 0 ? M - row0 : 0) : 32);
  int64_t ld = 0;
  const float* src = nullptr;
  if constexpr (kEpiReads<EPI>) src = epi_src<EPI>(ep, ld);
  auto step = [&](int c, float(&buf)[32]) {
    float v[32];
    ld32f(t_row + c, v);
#pragma unroll
    for (int i = 0; i < 32; ++i) wbuf[lane * 33 + i] = v[i];
    __syncwarp();
    const int64_t col = n0 + c + lane;
    const bool store = col < N && nrows > 0;
    const float* nsrc = nullptr;
    if constexpr (kEpiReads<EPI>) {
      if (c + 64 < BN && col + 64 < N && nrows > 0) nsrc = src + row0 * ld + col + 64;
    }
    if constexpr (EPI == EPI_SGD) {
      if (ep.c3)
        epi_chunk_check<EPI, true, true>(ep, row0, col, split, nrows, store, wbuf, buf, nsrc, ld);
      else if (ep.c2)
        epi_chunk_check<EPI, true, false>(ep, row0, col, split, nrows, store, wbuf, buf, nsrc, ld);
      else
        epi_chunk_check<EPI, false, false>(ep, row0, col, split, nrows, store, wbuf, buf, nsrc, ld);
    } else {
      epi_chunk_check<EPI, false, false>(ep, row0, col, split, nrows, store, wbuf, buf, nsrc, ld);
    }
    __syncwarp();
  };
  // one chunk per iteration: the two buffers alternate by branch, so that the
  // compiler cannot overlap two chunks' accumulator registers
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    if ((c & 32) == 0)
      step(c, bufA);
    else
      step(c, bufB);
  }
}

// Vectorised SGD epilogue of a warp's full 32 x BN tile (every row and
// column inside the output; master rows 16-byte aligned, hi/lo rows 8-byte
// aligned).  Per 32-column chunk, step it = 0..7 gives lane l row
// 4*it + l/8 and columns 4*(l%8) .. +3: one float4 read of the transposed
// accumulator, one float4 load (read ahead) and store of the master, one
// 8-byte store each of hi and lo.  The arithmetic per element is that of
// the scalar path: w = m - alpha*g, hi = bf16(w), lo = bf16(w - hi).
template <int EPI>
__device__ __forceinline__ bool sgd_vec_ok(const EpiArgs& ep, int64_t row0, int64_t M, int64_t n0, int64_t N,
                                           int bn) {
  if constexpr (EPI != EPI_SGD) {
    return false;
  } else {
    const bool m_ok = (reinterpret_cast<uintptr_t>(ep.c) & 15) == 0 && (ep.ldc & 3) == 0;
    const bool h_ok = !ep.c2 || ((reinterpret_cast<uintptr_t>(ep.c2) & 7) == 0 && (ep.ldc2 & 3) == 0);
    const bool l_ok = !ep.c3 || ((reinterpret_cast<uintptr_t>(ep.c3) & 7) == 0 && (ep.ldc3 & 3) == 0);
    return row0 + 32 <= M && n0 + bn <= N && m_ok && h_ok && l_ok;
  }
}

// L2 prefetch of the warp tile's master rows (lane l: row row0 + l, all bn
// columns, one request per 128-byte line), issued before the accumulator is
// ready: the tile's loads then find the master in L2 instead of waiting out a
// DRAM round trip two chunks at a time.
__device__ __forceinline__ void sgd_prefetch_tile(const EpiArgs& ep, int64_t row0, int64_t n0, int bn) {
  const int lane = threadIdx.x & 31;
  const float* p = reinterpret_cast<const float*>(ep.c) + (row0 + lane) * ep.ldc + n0;
  for (int c = 0; c < bn; c += 32) asm volatile("prefetch.global.L2 [%0];" ::"l"(p + c));
}

// Master values of one 32-column chunk in the vectorised layout.
__device__ __forceinline__ void sgd_load_vec(const EpiArgs& ep, int64_t row0, int64_t col0, float (&buf)[32]) {
  const int lane = threadIdx.x & 31;
  const float* p = reinterpret_cast<const float*>(ep.c) + (row0 + (lane >> 3)) * ep.ldc + col0 + 4 * (lane & 7);
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const float4 x = *reinterpret_cast<const float4*>(p + 4 * it * ep.ldc);
    buf[4 * it] = x.x;
    buf[4 * it + 1] = x.y;
    buf[4 * it + 2] = x.z;
    buf[4 * it + 3] = x.w;
  }
}

__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}

template <bool HI, bool LO>
__device__ __forceinline__ void sgd_chunk_vec(const EpiArgs& ep, int64_t row0, int64_t col0, bool ahead,
                                              const float* wbuf, float (&buf)[32]) {
  const int lane = threadIdx.x & 31;
  const int rs = lane >> 3, c4 = 4 * (lane & 7);
  float* pm = reinterpret_cast<float*>(ep.c) + (row0 + rs) * ep.ldc + col0 + c4;
  bf16* ph = HI ? reinterpret_cast<bf16*>(ep.c2) + (row0 + rs) * ep.ldc2 + col0 + c4 : nullptr;
  bf16* pl = LO ? reinterpret_cast<bf16*>(ep.c3) + (row0 + rs) * ep.ldc3 + col0 + c4 : nullptr;
  const float na = -ep.alpha;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const float4 g = *reinterpret_cast<const float4*>(wbuf + (4 * it + rs) * 36 + c4);
    const float w0 = __fmaf_rn(na, g.x, buf[4 * it]), w1 = __fmaf_rn(na, g.y, buf[4 * it + 1]);
    const float w2 = __fmaf_rn(na, g.z, buf[4 * it + 2]), w3 = __fmaf_rn(na, g.w, buf[4 * it + 3]);
    float* m = pm + (int64_t)(4 * it) * ep.ldc;
    *reinterpret_cast<float4*>(m) = make_float4(w0, w1, w2, w3);
    if constexpr (HI) {
      const uint32_t h01 = bf16x2_bits(w0, w1), h23 = bf16x2_bits(w2, w3);
      *reinterpret_cast<uint2*>(ph + (int64_t)(4 * it) * ep.ldc2) = make_uint2(h01, h23);
      if constexpr (LO) {
        const float f0 = __uint_as_float(h01 << 16), f1 = __uint_as_float(h01 & 0xFFFF0000u);
        const float f2 = __uint_as_float(h23 << 16), f3 = __uint_as_float(h23 & 0xFFFF0000u);
        *reinterpret_cast<uint2*>(pl + (int64_t)(4 * it) * ep.ldc3) =
            make_uint2(bf16x2_bits(w0 - f0, w1 - f1), bf16x2_bits(w2 - f2, w3 - f3));
      }
    }
    if (ahead) {  // the same rows, two chunks (64 columns) further on
      const float4 x = *reinterpret_cast<const float4*>(m + 64);
      buf[4 * it] = x.x;
      buf[4 * it + 1] = x.y;
      buf[4 * it + 2] = x.z;
      buf[4 * it + 3] = x.w;
    }
  }
}

// bufA / bufB hold the master of chunks 0 and 1 (sgd_load_vec) on entry.
template <int BN>
__device__ __forceinline__ void epilogue_sgd_vec(uint32_t t_row, const EpiArgs& ep, int64_t n0, float* wbuf,
                                                 int64_t row0, float (&bufA)[32], float (&bufB)[32]) {
  const int lane = threadIdx.x & 31;
  auto step = [&](int c, float(&buf)[32]) {
    float v[32];
    ld32f(t_row + c, v);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(wbuf + lane * 36 + 4 * j) = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2],
                                                                         v[4 * j + 3]);
    __syncwarp();
    const bool ahead = c + 64 < BN;
    if (ep.c3)
      sgd_chunk_vec<true, true>(ep, row0, n0 + c, ahead, wbuf, buf);
    else if (ep.c2)
      sgd_chunk_vec<true, false>(ep, row0, n0 + c, ahead, wbuf, buf);
    else
      sgd_chunk_vec<false, false>(ep, row0, n0 + c, ahead, wbuf, buf);
    __syncwarp();
  };
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    if ((c & 32) == 0)
      step(c, bufA);
    else
      step(c, bufB);
  }
}

// Persistent kernel: one CTA per SM walks the work units u = blockIdx.x,
// blockIdx.x + gridDim.x, ...  A unit is (m-tile, n-tile, k-split) with the
// m-tile fastest, so CTAs running at the same time share weight (B) tiles in
// L2.  The accumulator is double-buffered in TMEM (2 x BN columns): the
// epilogue warps drain unit i while the MMA thread already accumulates unit
// i+1.  The smem ring's stage/phase counters run on across units.
//
// Second product: output tiles with n0 >= n_ext accumulate A2 B2^T after
// A B^T (k-blocks KB1 .. KB1+KB2-1 of the concatenated reduction; B2's row is
// n0 - n_ext).  The k-splits cut the concatenated range.
// Output tile (m-tile, n-tile) of linear index mn.  raster 0: m-tile fastest;
// 1: n-tile fastest; raster >= 2: groups of `raster` m-tiles walked m-tile
// fastest, one n-tile after the other, so that while the resident units
// cover a group, its rows of A and the current columns of B both stay in L2
// (for products whose A and B are each larger than a third of L2).
__device__ __forceinline__ void tile_of(int64_t mn, int n_mt, int n_nt, int raster, int64_t& mt, int64_t& nt) {
  if (raster == 0) {
    mt = mn % n_mt;
    nt = mn / n_mt;
  } else if (raster == 1) {
    mt = mn / n_nt;
    nt = mn % n_nt;
  } else {
    const int64_t per_group = (int64_t)raster * n_nt;
    const int64_t m_first = (mn / per_group) * raster, r = mn % per_group;
    const int64_t gm = imin64(raster, n_mt - m_first);  // the last group may hold fewer m-tiles
    mt = m_first + r % gm;
    nt = r / gm;
  }
}

template <int BN, bool A_MN, bool B_MN, int EPI, typename TACT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
                   const __grid_constant__ CUtensorMap tma2, const __grid_constant__ CUtensorMap tmb2, int64_t M,
                   int64_t N, int KB1, int KB2, int64_t n_ext, int kpsb, int n_mt, int n_nt, int n_split, int n_fast,
                   EpiArgs ep,
                   int* err) {
  using C = TcCfg<BN, EPI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  float* wbufs = reinterpret_cast<float*>(sB + C::STAGES * C::B_BYTES + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t units = (int64_t)n_mt * n_nt * n_split;
  // k-blocks [kb_begin, kb_begin + nkb) of this unit's concatenated reduction
  // Raster: m-tile fastest (CTAs running together share B tiles: large weights,
  // few rows) or n-tile fastest (they share A tiles: B small enough to stay in
  // L2 while A streams through once).
  auto decode = [&](int64_t u, int64_t& m0, int64_t& n0, int& split, int& nkb, int& kb_begin) {
    const int64_t mn = u % ((int64_t)n_mt * n_nt);
    int64_t mt, nt;
    tile_of(mn, n_mt, n_nt, n_fast, mt, nt);
    m0 = mt * BM;
    n0 = nt * BN;
    split = (int)(u / ((int64_t)n_mt * n_nt));
    const int total = KB1 + (n0 >= n_ext ? KB2 : 0);
    kb_begin = split * kpsb;
    nkb = total - kb_begin < kpsb ? total - kb_begin : kpsb;
    if (nkb < 0) nkb = 0;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&acc_full[b], 1);
      ptx::mbar_init(&acc_empty[b], 128);
    }
    ptx::mbar_init(drain, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tma);
    ptx::prefetch_tmap(&tmb);
    if (KB2 > 0) {
      ptx::prefetch_tmap(&tma2);
      ptx::prefetch_tmap(&tmb2);
    }
  }
  if (warp == 1) {
    __syncwarp();
    ptx::tmem_alloc(tmem_slot, 2 * BN);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    {  // the converged warp polls the ring; lane 0 issues the loads
      uint32_t kbg = 0;  // k-blocks issued by this CTA so far (ring position)
      bool ok = true;
      for (int64_t u = blockIdx.x; ok && u < units; u += gridDim.x) {
        int64_t m0, n0;
        int split, nkb, kb_begin;
        decode(u, m0, n0, split, nkb, kb_begin);
        for (int j = 0; j < nkb; ++j, ++kbg) {
          const int s = (int)(kbg % C::STAGES);
          const uint32_t ph = (kbg / C::STAGES) & 1u;
          if (!(ok = ptx::mbar_wait_warp(&empty[s], ph ^ 1u, err))) break;
          if (lane != 0) continue;
          ptx::mbar_arrive_expect_tx(&full[s], C::STAGE);
          uint8_t* a = sA + s * C::A_BYTES;
          uint8_t* b = sB + s * C::B_BYTES;
          const int kb = kb_begin + j;
          const bool second = kb >= KB1;  // block of the second product
          const CUtensorMap* ta = second ? &tma2 : &tma;
          const CUtensorMap* tb = second ? &tmb2 : &tmb;
          const int k0 = (second ? kb - KB1 : kb) * BK;
          const int nb = (int)(second ? n0 - n_ext : n0);
          if constexpr (!A_MN) {
            ptx::tma_load_2d(a, ta, &full[s], k0, (int)m0);
          } else {
            ptx::tma_load_2d(a, ta, &full[s], (int)m0, k0);
            ptx::tma_load_2d(a + 8192, ta, &full[s], (int)m0 + 64, k0);
          }
          if constexpr (!B_MN) {
            ptx::tma_load_2d(b, tb, &full[s], k0, nb);
          } else {
#pragma unroll
            for (int jj = 0; jj < BN / 64; ++jj) ptx::tma_load_2d(b + jj * 8192, tb, &full[s], nb + 64 * jj, k0);
          }
        }
      }
    }
  } else if (warp == 1) {
    {  // the converged warp runs the issue loop; one elected lane issues each MMA and commit
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(BM, BN, A_MN, B_MN);
      uint32_t kbg = 0, it = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; ok && u < units; u += gridDim.x, ++it) {
        int64_t m0, n0;
        int split, nkb, kb_begin;
        decode(u, m0, n0, split, nkb, kb_begin);
        const uint32_t b = it & 1u, use = it >> 1;
        // the epilogue must have drained this accumulator buffer's previous unit
        if (!(ok = ptx::mbar_wait_warp(&acc_empty[b], (use & 1u) ^ 1u, err))) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + b * BN;
        for (int kb = 0; kb < nkb; ++kb, ++kbg) {
          const int s = (int)(kbg % C::STAGES);
          const uint32_t ph = (kbg / C::STAGES) & 1u;
          if (!(ok = ptx::mbar_wait_warp(&full[s], ph, err))) break;
          ptx::tc_fence_after();
          const uint32_t a_addr = ptx::smem_u32(sA + s * C::A_BYTES);
          const uint32_t b_addr = ptx::smem_u32(sB + s * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = A_MN ? ptx::smem_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                     : ptx::smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? ptx::smem_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                     : ptx::smem_desc_sw128(b_addr + kk * 32, 16, 1024);
            ptx::umma_bf16_elect(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          ptx::umma_commit_elect(&empty[s]);
        }
        if (!ok) break;
        ptx::umma_commit_elect(&acc_full[b]);
      }
      // Arrives once every MMA issued above has completed (also on a bail-out).
      ptx::umma_commit_elect(drain);
      ptx::mbar_drain(drain, 0);  // no MMA may still write TMEM when it is released
    }
  } else {
    // epilogue group eg drains accumulator buffer eg: the units with it = eg, eg + 2, ...
    const int ew = warp - 2, eg = ew >> 2;
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint32_t it = (uint32_t)eg;
    for (int64_t u = blockIdx.x + (int64_t)eg * gridDim.x; u < units; u += 2 * (int64_t)gridDim.x, it += 2) {
      int64_t m0, n0;
      int split, nkb, kb_begin;
      decode(u, m0, n0, split, nkb, kb_begin);
      const uint32_t b = it & 1u, use = it >> 1;
      float bufA[32], bufB[32];
      const bool vec = sgd_vec_ok<EPI>(ep, m0 + q * 32, M, n0, N, BN);  // warp-uniform
      if constexpr (kTransposedEpi<EPI>) {  // read source of the first two chunks, ahead of the accumulator
        if (vec) {
          sgd_prefetch_tile(ep, m0 + q * 32, n0, BN);
          sgd_load_vec(ep, m0 + q * 32, n0, bufA);
          sgd_load_vec(ep, m0 + q * 32, n0 + 32, bufB);
        } else {
          epi_load_chunk<EPI>(ep, m0 + q * 32, M, n0 + lane, N, bufA);
          epi_load_chunk<EPI>(ep, m0 + q * 32, M, n0 + 32 + lane, N, bufB);
        }
      }
      const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(&acc_full[b], use & 1u, err));  // warp-uniform
      if (!ok) break;
      ptx::tc_fence_after();
      const int64_t row = m0 + q * 32 + lane;
      if constexpr (EPI == EPI_SGD) {
        if (vec)
          epilogue_sgd_vec<BN>(tmem + b * BN + lane_off, ep, n0, wbufs + ew * 32 * kWStride<EPI>, m0 + q * 32, bufA,
                               bufB);
        else
          epilogue_transposed<BN, EPI>(tmem + b * BN + lane_off, ep, n0, N, split, wbufs + ew * 32 * kWStride<EPI>,
                                       m0 + q * 32, M, bufA, bufB);
      } else if constexpr (kTransposedEpi<EPI>)
        epilogue_transposed<BN, EPI>(tmem + b * BN + lane_off, ep, n0, N, split, wbufs + ew * 32 * kWStride<EPI>, m0 + q * 32,
                                     M, bufA, bufB);
      else
        epilogue_row<BN, EPI, TACT>(tmem + b * BN + lane_off, row, row < M, n0, N, ep, (int)(n0 / BN), split);
      ptx::tc_fence_before();
      ptx::mbar_arrive(&acc_empty[b]);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();  // tcgen05.dealloc is warp-collective: reconverge lane 0 with the others
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 2 * BN);
  }
}

// CTA-pair variant: a cluster of two CTAs (two SMs) computes one 256 x BN
// output tile (BN = 256 or 128) with tcgen05.mma.cta_group::2.  Each CTA
// loads its own 128 rows of A and its half (BN/2 rows) of the B tile: for
// BN = 256, 32 KB per 64-deep k-block instead of the 48 KB a single CTA needs
// for a 128 x 256 tile, so a CTA streams 131 instead of 87 flop per operand
// byte.  A pair MMA also runs at the tensor cores' rate for N = 128 (about 65
// cycles per 16-deep step, measured), where a single-CTA M = 128 MMA costs
// about 100 cycles whatever its N up to 128: the narrow tiles of the
// M = b products therefore run on pairs as well.  Roles:
//   even CTA, warp 0 lane 0   TMA for its halves; arrives on its own full
//                             barrier with the bytes of both CTAs
//   odd CTA,  warp 0 lane 0   TMA for its halves, counted on the even CTA's
//                             full barrier
//   even CTA, warp 1 lane 0   issues every MMA of the pair; each commit frees
//                             the ring slot / fills the accumulator in both
//                             CTAs at once
//   warps 2..9 (both CTAs)    epilogue of the CTA's own 128 accumulator rows,
//                             then an arrive on the even CTA's acc_empty
//                             (256 arrivals: both CTAs' epilogue groups)
// The units are (256-row pair tile, n-tile, k-split), walked by the pairs
// like the single-CTA kernel walks its tiles.
template <int EPI, int BN_, bool B_MN>
struct PairCfg {
  static constexpr int BN = BN_;
  static constexpr int A_BYTES = BM * BK * 2;  // this CTA's 128 rows of A
  // this CTA's half of the B tile: BN/2 rows (K-major), or BN/2 columns in
  // whole 64-column boxes (MN-major)
  static constexpr int NBOX = (BN / 2 + 63) / 64;
  static constexpr int B_BYTES = B_MN ? NBOX * 64 * BK * 2 : (BN / 2) * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int WBUF = kEpiWarps * 32 * kWStride<EPI> * 4;
  static constexpr int STAGES_FIT = (232448 - 1024 - 256 - WBUF) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int SMEM = STAGES * STAGE + 1024 + 256 + WBUF;
  // TMEM: two accumulator buffers of BN columns, allocated as a power of two
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static_assert(B_BYTES % 1024 == 0, "1024-byte aligned B stages");
  static_assert(SMEM <= 232448, "shared memory per block");
};

template <int BN_, bool A_MN, bool B_MN, int EPI, typename TACT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
                        const __grid_constant__ CUtensorMap tma2, const __grid_constant__ CUtensorMap tmb2,
                        int64_t M, int64_t N, int KB1, int KB2, int64_t n_ext, int kpsb, int n_mt, int n_nt,
                        int n_split, int n_fast, EpiArgs ep, int* err) {
  using C = PairCfg<EPI, BN_, B_MN>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2], used in the even CTA
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  float* wbufs = reinterpret_cast<float*>(sB + C::STAGES * C::B_BYTES + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();  // 0: issues the MMAs
  const bool lead = rank == 0;
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int64_t units = (int64_t)n_mt * n_nt * n_split;
  // n_mt counts 256-row pair tiles; m0 is the pair tile's first row
  auto decode = [&](int64_t u, int64_t& m0, int64_t& n0, int& split, int& nkb, int& kb_begin) {
    const int64_t mn = u % ((int64_t)n_mt * n_nt);
    int64_t mt, nt;
    tile_of(mn, n_mt, n_nt, n_fast, mt, nt);
    m0 = mt * (2 * BM);
    n0 = nt * BN;
    split = (int)(u / ((int64_t)n_mt * n_nt));
    const int total = KB1 + (n0 >= n_ext ? KB2 : 0);
    kb_begin = split * kpsb;
    nkb = total - kb_begin < kpsb ? total - kb_begin : kpsb;
    if (nkb < 0) nkb = 0;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&acc_full[b], 1);
      ptx::mbar_init(&acc_empty[b], 256);
    }
    ptx::mbar_init(drain, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tma);
    ptx::prefetch_tmap(&tmb);
    if (KB2 > 0) {
      ptx::prefetch_tmap(&tma2);
      ptx::prefetch_tmap(&tmb2);
    }
  }
  if (warp == 1) {
    __syncwarp();
    ptx::tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync_all();  // both CTAs' barriers are initialised before either signals the other
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    {  // the converged warp polls the ring; lanes 0 .. NLOADS-1 issue the stage's boxes together
      constexpr int NA = A_MN ? 2 : 1;
      constexpr int NLOADS = NA + (B_MN ? C::NBOX : 1);
      const uint32_t fb0 = ptx::mapa_shared(ptx::smem_u32(&full[0]), 0);
      uint32_t kbg = 0;
      bool ok = true;
      for (int64_t u = pair; ok && u < units; u += npairs) {
        int64_t m0, n0;
        int split, nkb, kb_begin;
        decode(u, m0, n0, split, nkb, kb_begin);
        const int mo = (int)(m0 + BM * rank);  // this CTA's A rows
        for (int j = 0; j < nkb; ++j, ++kbg) {
          const int s = (int)(kbg % C::STAGES);
          const uint32_t ph = (kbg / C::STAGES) & 1u;
          if (!(ok = ptx::mbar_wait_warp(&empty[s], ph ^ 1u, err))) break;
          // one lane per box, all boxes of the stage in one TMA instruction of the warp: a
          // TMA instruction costs its issuing thread about 125 cycles (measured), so issuing
          // the boxes one after another from lane 0 made the producer, not the MMAs, set the
          // pace of the narrow-tile products
          if (lane >= NLOADS) continue;
          if (lane == 0 && lead) ptx::mbar_arrive_expect_tx(&full[s], 2 * C::STAGE);
          const uint32_t fb = fb0 + 8u * (uint32_t)s;  // &full[s] in the even CTA
          const int kb = kb_begin + j;
          const bool second = kb >= KB1;
          const int k0 = (second ? kb - KB1 : kb) * BK;
          const int nb = (int)(second ? n0 - n_ext : n0) + (BN / 2) * (int)rank;  // this CTA's half of B
          uint8_t* dst;
          const CUtensorMap* tm;
          int c0, c1;
          if (lane < NA) {  // A: this CTA's 128 rows (K-major: one box; MN-major: two 64-row boxes)
            dst = sA + s * C::A_BYTES + 8192 * lane;
            tm = second ? &tma2 : &tma;
            c0 = A_MN ? mo + 64 * lane : k0;
            c1 = A_MN ? k0 : mo;
          } else {  // B: this CTA's half (K-major: one box; MN-major: NBOX 64-column boxes)
            const int i = lane - NA;
            dst = sB + s * C::B_BYTES + 8192 * i;
            tm = second ? &tmb2 : &tmb;
            c0 = B_MN ? nb + 64 * i : k0;
            c1 = B_MN ? k0 : nb;
          }
          ptx::tma_load_2d_pair(dst, tm, fb, c0, c1);
        }
      }
    }
  } else if (warp == 1) {
    {  // the converged warp runs the issue loop; one elected lane issues each MMA and commit
      if (lead) {
        constexpr uint32_t idesc = ptx::idesc_bf16_f32(2 * BM, BN, A_MN, B_MN);
        uint32_t kbg = 0, it = 0;
        bool ok = true;
        for (int64_t u = pair; ok && u < units; u += npairs, ++it) {
          int64_t m0, n0;
          int split, nkb, kb_begin;
          decode(u, m0, n0, split, nkb, kb_begin);
          const uint32_t b = it & 1u, use = it >> 1;
          // both CTAs' epilogues must have drained this accumulator buffer
          if (!(ok = ptx::mbar_wait_warp(&acc_empty[b], (use & 1u) ^ 1u, err))) break;
          ptx::tc_fence_after();
          const uint32_t d_tmem = tmem + b * BN;
          for (int kb = 0; kb < nkb; ++kb, ++kbg) {
            const int s = (int)(kbg % C::STAGES);
            const uint32_t ph = (kbg / C::STAGES) & 1u;
            if (!(ok = ptx::mbar_wait_warp(&full[s], ph, err))) break;
            ptx::tc_fence_after();
            const uint32_t a_addr = ptx::smem_u32(sA + s * C::A_BYTES);
            const uint32_t b_addr = ptx::smem_u32(sB + s * C::B_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = A_MN ? ptx::smem_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                       : ptx::smem_desc_sw128(a_addr + kk * 32, 16, 1024);
              const uint64_t bd = B_MN ? ptx::smem_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                       : ptx::smem_desc_sw128(b_addr + kk * 32, 16, 1024);
              ptx::umma_bf16_pair_elect(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            ptx::umma_commit_pair_elect(&empty[s], 0x3);
          }
          if (!ok) break;
          ptx::umma_commit_pair_elect(&acc_full[b], 0x3);
        }
        ptx::umma_commit_pair_elect(drain, 0x3);
      }
      // every MMA of the pair has completed (they read this CTA's shared
      // memory and write its TMEM) before either CTA releases them
      ptx::mbar_drain(drain, 0);
    }
  } else {
    const int ew = warp - 2, eg = ew >> 2;
    const int q = warp & 3;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t empty_lead0 = ptx::mapa_shared(ptx::smem_u32(&acc_empty[0]), 0);
    const uint32_t empty_lead1 = ptx::mapa_shared(ptx::smem_u32(&acc_empty[1]), 0);
    uint32_t it = (uint32_t)eg;
    for (int64_t u = pair + (int64_t)eg * npairs; u < units; u += 2 * npairs, it += 2) {
      int64_t m0, n0;
      int split, nkb, kb_begin;
      decode(u, m0, n0, split, nkb, kb_begin);
      m0 += BM * rank;  // this CTA's 128 rows of the pair tile
      const uint32_t b = it & 1u, use = it >> 1;
      float bufA[32], bufB[32];
      const bool vec = sgd_vec_ok<EPI>(ep, m0 + q * 32, M, n0, N, BN);  // warp-uniform
      if constexpr (kTransposedEpi<EPI>) {
        if (vec) {
          sgd_prefetch_tile(ep, m0 + q * 32, n0, BN);
          sgd_load_vec(ep, m0 + q * 32, n0, bufA);
          sgd_load_vec(ep, m0 + q * 32, n0 + 32, bufB);
        } else {
          epi_load_chunk<EPI>(ep, m0 + q * 32, M, n0 + lane, N, bufA);
          epi_load_chunk<EPI>(ep, m0 + q * 32, M, n0 + 32 + lane, N, bufB);
        }
      }
      const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(&acc_full[b], use & 1u, err));
      if (!ok) break;
      ptx::tc_fence_after();
      const int64_t row = m0 + q * 32 + lane;
      if constexpr (EPI == EPI_SGD) {
        if (vec)
          epilogue_sgd_vec<BN>(tmem + b * BN + lane_off, ep, n0, wbufs + ew * 32 * kWStride<EPI>, m0 + q * 32, bufA,
                               bufB);
        else
          epilogue_transposed<BN, EPI>(tmem + b * BN + lane_off, ep, n0, N, split, wbufs + ew * 32 * kWStride<EPI>,
                                       m0 + q * 32, M, bufA, bufB);
      } else if constexpr (kTransposedEpi<EPI>)
        epilogue_transposed<BN, EPI>(tmem + b * BN + lane_off, ep, n0, N, split, wbufs + ew * 32 * kWStride<EPI>, m0 + q * 32,
                                     M, bufA, bufB);
      else
        epilogue_row<BN, EPI, TACT>(tmem + b * BN + lane_off, row, row < M, n0, N, ep, (int)(n0 / BN), split);
      ptx::tc_fence_before();
      ptx::mbar_arrive_cluster(b ? empty_lead1 : empty_lead0);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync_all();  // neither CTA frees TMEM or exits while the pair still uses it
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

// ---- host side -----------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 row-major [rows, cols] (leading dim ld elements), box = 64 cols x box_rows rows, 128B swizzle.
int make_tmap(CUtensorMap* tm, const MatView& v, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return set_error(TTT_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  if ((reinterpret_cast<uintptr_t>(v.ptr) & 15) || ((v.ld * 2) & 15) || v.rows < 1 || v.cols < 1 || v.ld < v.cols)
    return set_error(TTT_ERR_INVALID_ARG, "TMA operand must be 16-byte aligned with a 16-byte multiple row pitch");
  cuuint64_t dims[2] = {(cuuint64_t)v.cols, (cuuint64_t)v.rows};
  cuuint64_t strides[1] = {(cuuint64_t)(v.ld * 2)};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(v.ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(TTT_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return TTT_OK;
}

using KernelFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, int64_t, int64_t, int, int, int64_t, int,
                          int, int, int, int, EpiArgs, int*);

// Sum of split-K partials in a fixed order (deterministic), then the epilogue.
// A thread owns 4 consecutive columns of one row; when they are 16-byte aligned
// and all inside the row, the S partials are read as float4, all loads issued
// before the (in-order) sum so that up to 8 are in flight per thread.
template <int EPI>
__device__ __forceinline__ void splitk_out(const EpiArgs& ep, int64_t row, int64_t col, const float* v, int cnt) {
  if constexpr (EPI == EPI_STORE_F32 || EPI == EPI_ADD_F32) {
    float* dst = reinterpret_cast<float*>(ep.c) + row * ep.ldc + col;
    const float* res = nullptr;
    if constexpr (EPI == EPI_ADD_F32)
      res = ep.c2 ? reinterpret_cast<const float*>(ep.c2) + row * ep.ldc2 + col : dst;
    const bool vec = cnt == 4 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0 &&
                     (EPI != EPI_ADD_F32 || (reinterpret_cast<uintptr_t>(res) & 15) == 0);
    if (vec) {
      float4 o = make_float4(v[0], v[1], v[2], v[3]);
      if constexpr (EPI == EPI_ADD_F32) {
        const float4 r = *reinterpret_cast<const float4*>(res);
        o = make_float4(r.x + v[0], r.y + v[1], r.z + v[2], r.w + v[3]);
      }
      *reinterpret_cast<float4*>(dst) = o;
      return;
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (e >= cnt) break;
    if constexpr (EPI == EPI_STORE_F32) {
      reinterpret_cast<float*>(ep.c)[row * ep.ldc + col + e] = v[e];
    } else if constexpr (EPI == EPI_STORE_BF16) {
      reinterpret_cast<bf16*>(ep.c)[row * ep.ldc + col + e] = __float2bfloat16_rn(v[e]);
    } else {  // EPI_ADD_F32
      const float r = ep.c2 ? reinterpret_cast<const float*>(ep.c2)[row * ep.ldc2 + col + e]
                            : reinterpret_cast<const float*>(ep.c)[row * ep.ldc + col + e];
      reinterpret_cast<float*>(ep.c)[row * ep.ldc + col + e] = r + v[e];
    }
  }
}

template <int EPI>
__global__ void splitk_reduce_kernel(const float* __restrict__ ws, int S, int64_t M, int64_t N, int64_t stride,
                                     EpiArgs ep) {
  const int64_t gpr = (N + 3) / 4;  // 4-column groups per row
  const int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gi >= M * gpr) return;
  const int64_t row = gi / gpr, col = (gi % gpr) * 4;
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  const int cnt = (int)imin64(4, N - col);
  const float* p0 = ws + row * N + col;
  if (cnt == 4 && (reinterpret_cast<uintptr_t>(p0) & 15) == 0 && (stride & 3) == 0 && S <= 8) {
    float4 part[8];
#pragma unroll
    for (int s = 0; s < 8; ++s)
      if (s < S) part[s] = *reinterpret_cast<const float4*>(p0 + s * stride);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      if (s < S) {
        v[0] += part[s].x;
        v[1] += part[s].y;
        v[2] += part[s].z;
        v[3] += part[s].w;
      }
    }
  } else {
    for (int s = 0; s < S; ++s) {
      const float* p = p0 + s * stride;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (e < cnt) v[e] += p[e];
    }
  }
  splitk_out<EPI>(ep, row, col, v, cnt);
}

template <int BN, bool A_MN, bool B_MN, int EPI, typename TACT>
KernelFn kernel_ptr() {
  return reinterpret_cast<KernelFn>(&tc_gemm_kernel<BN, A_MN, B_MN, EPI, TACT>);
}

template <int BN, bool A_MN, bool B_MN>
KernelFn pick_epi(int epi, int act_bf16) {
  switch (epi) {
    case EPI_STORE_F32: return kernel_ptr<BN, A_MN, B_MN, EPI_STORE_F32, bf16>();
    case EPI_STORE_BF16: return kernel_ptr<BN, A_MN, B_MN, EPI_STORE_BF16, bf16>();
    case EPI_ADD_F32: return kernel_ptr<BN, A_MN, B_MN, EPI_ADD_F32, bf16>();
    case EPI_SWIGLU:
      return act_bf16 ? kernel_ptr<BN, A_MN, B_MN, EPI_SWIGLU, bf16>() : kernel_ptr<BN, A_MN, B_MN, EPI_SWIGLU, float>();
    case EPI_CE_FWD: return kernel_ptr<BN, A_MN, B_MN, EPI_CE_FWD, bf16>();
    case EPI_CE_BWD:
      return act_bf16 ? kernel_ptr<BN, A_MN, B_MN, EPI_CE_BWD, bf16>() : kernel_ptr<BN, A_MN, B_MN, EPI_CE_BWD, float>();
    case EPI_SGD: return kernel_ptr<BN, A_MN, B_MN, EPI_SGD, bf16>();
  }
  return nullptr;
}

template <int BN, bool A_MN, bool B_MN, int EPI, typename TACT>
KernelFn pair_ptr() {
  return reinterpret_cast<KernelFn>(&tc_gemm_pair_kernel<BN, A_MN, B_MN, EPI, TACT>);
}

template <int BN, bool A_MN, bool B_MN>
KernelFn pick_pair_epi(int epi, int act_bf16) {
  if constexpr (BN == 160) {  // 160-wide tiles: plain stores and the residual add only
    switch (epi) {
      case EPI_STORE_F32: return pair_ptr<BN, A_MN, B_MN, EPI_STORE_F32, bf16>();
      case EPI_STORE_BF16: return pair_ptr<BN, A_MN, B_MN, EPI_STORE_BF16, bf16>();
      case EPI_ADD_F32: return pair_ptr<BN, A_MN, B_MN, EPI_ADD_F32, bf16>();
    }
    return nullptr;
  }
  switch (epi) {
    case EPI_STORE_F32: return pair_ptr<BN, A_MN, B_MN, EPI_STORE_F32, bf16>();
    case EPI_STORE_BF16: return pair_ptr<BN, A_MN, B_MN, EPI_STORE_BF16, bf16>();
    case EPI_ADD_F32: return pair_ptr<BN, A_MN, B_MN, EPI_ADD_F32, bf16>();
    case EPI_SWIGLU:
      return act_bf16 ? pair_ptr<BN, A_MN, B_MN, EPI_SWIGLU, bf16>() : pair_ptr<BN, A_MN, B_MN, EPI_SWIGLU, float>();
    case EPI_CE_FWD: return pair_ptr<BN, A_MN, B_MN, EPI_CE_FWD, bf16>();
    case EPI_CE_BWD:
      return act_bf16 ? pair_ptr<BN, A_MN, B_MN, EPI_CE_BWD, bf16>() : pair_ptr<BN, A_MN, B_MN, EPI_CE_BWD, float>();
    case EPI_SGD: return pair_ptr<BN, A_MN, B_MN, EPI_SGD, bf16>();
  }
  return nullptr;
}

template <int BN>
KernelFn pick_pair_bn(int a_mn, int b_mn, int epi, int act_bf16) {
  if (!a_mn && !b_mn) return pick_pair_epi<BN, false, false>(epi, act_bf16);
  if (!a_mn && b_mn) return pick_pair_epi<BN, false, true>(epi, act_bf16);
  if (a_mn && b_mn) return pick_pair_epi<BN, true, true>(epi, act_bf16);
  return pick_pair_epi<BN, true, false>(epi, act_bf16);
}

KernelFn pick_pair(int bn, int a_mn, int b_mn, int epi, int act_bf16) {
  switch (bn) {
    case 256: return pick_pair_bn<256>(a_mn, b_mn, epi, act_bf16);
    case 160: return pick_pair_bn<160>(a_mn, b_mn, epi, act_bf16);
    case 128: return pick_pair_bn<128>(a_mn, b_mn, epi, act_bf16);
  }
  return nullptr;
}

// CTA pairs for every GEMM with more than one 128-row tile;
// TTT_GEMM_PAIR=0 keeps every GEMM on single CTAs.
bool pair_enabled() {
  static const bool on = [] {
    const char* e = getenv("TTT_GEMM_PAIR");
    return !(e && e[0] == '0');
  }();
  return on;
}

template <int BN>
KernelFn pick(int a_mn, int b_mn, int epi, int act_bf16) {
  if (!a_mn && !b_mn) return pick_epi<BN, false, false>(epi, act_bf16);
  if (!a_mn && b_mn) return pick_epi<BN, false, true>(epi, act_bf16);
  if (a_mn && b_mn) return pick_epi<BN, true, true>(epi, act_bf16);
  return pick_epi<BN, true, false>(epi, act_bf16);
}

template <int EPI, bool B_MN>
int pair_smem(int bn) {
  return bn == 256 ? PairCfg<EPI, 256, B_MN>::SMEM
                   : (bn == 160 ? PairCfg<EPI, 160, B_MN>::SMEM : PairCfg<EPI, 128, B_MN>::SMEM);
}

template <int EPI>
int smem_bytes_epi(int pair, int bn, int b_mn) {
  if (pair) return b_mn ? pair_smem<EPI, true>(bn) : pair_smem<EPI, false>(bn);
  return bn == 256 ? TcCfg<256, EPI>::SMEM : TcCfg<128, EPI>::SMEM;
}

int smem_bytes(int pair, int bn, int epi, int b_mn) {
  return epi == EPI_SGD ? smem_bytes_epi<EPI_SGD>(pair, bn, b_mn) : smem_bytes_epi<EPI_STORE_F32>(pair, bn, b_mn);
}

}  // namespace

int64_t tc_ce_tiles(int64_t N, int bn) { return (N + bn - 1) / bn; }

int tc_pick_bn(int64_t M, int64_t N, int hint) {
  if (hint == 128 || hint == 160 || hint == 256) return hint;
  // Prefer 256-wide tiles when that still gives every SM a tile.
  const int64_t tiles256 = ((N + 255) / 256) * ((M + BM - 1) / BM);
  return (tiles256 >= 148 || N > 4096) ? 256 : 128;
}

namespace {
// Cost (cycles) of a store/add GEMM on CTA pairs with bn-wide tiles and S
// splits of K, fitted to measured b-row products (M = 1024, N = 2560, K from
// 2560 to 27648, tile widths 128 to 256, 1 to 6 splits): every pair slot
// runs ceil(units / slots) work units one after the other; a unit costs
// about 13000 cycles of start, pipeline fill and epilogue plus about 760
// cycles per 64-deep k-block (whatever the tile width: the operand pipeline,
// not the tensor core, sets that pace), or its four pair MMAs if slower;
// split-K adds about 30000 cycles for the partials' round trip through HBM
// and the reduction launch.  Only the ranking matters.
double pair_cost(int64_t M, int64_t N, int64_t K, int bn, int64_t S) {
  const int64_t slots = 74;
  const int64_t tiles = ((M + 2 * BM - 1) / (2 * BM)) * ((N + bn - 1) / bn);
  const int64_t units = tiles * S;
  const int64_t waves = (units + slots - 1) / slots;
  const int64_t kb = ((K + BK - 1) / BK + S - 1) / S;
  const double per_kb = std::max(4.0 * (bn / 2 + 1), 760.0);
  double t = (double)waves * ((double)kb * per_kb + 13000.0);
  if (S > 1) t += 30000.0 + (double)(S + 1) * (double)M * (double)N * 4.0 / 3600.0;
  return t;
}
}  // namespace

int64_t tc_split_plan(int64_t M, int64_t N, int64_t K, int epi, int* bn_out) {
  *bn_out = 0;
  if (epi != EPI_STORE_F32 && epi != EPI_STORE_BF16 && epi != EPI_ADD_F32) return 1;
  if (M > BM && pair_enabled()) {
    // CTA pairs: the tile width (160, 256 or 128) and split count (1..8, at
    // least 16 k-blocks each) of least modelled cost; an earlier width or
    // fewer splits must lose by more than 3% to be passed over.
    const int64_t kb = (K + BK - 1) / BK;
    double best = 0.0;
    int best_bn = 0;
    int64_t best_s = 1;
    for (int bn : {160, 256, 128}) {
      for (int64_t S = 1; S <= 8; ++S) {
        if (S > 1 && kb / S < 16) break;
        const double c = pair_cost(M, N, K, bn, S);
        if (best_bn == 0 || c < 0.97 * best) {
          best = c;
          best_bn = bn;
          best_s = S;
        }
      }
    }
    *bn_out = best_bn;
    return best_s;
  }
  // Single CTAs: split K when the output alone gives fewer than two waves of
  // 256-wide tiles and the reduction is long: pick the split count (2..8,
  // >= 1024 of K each) whose work units fill the 148 SMs best.
  const int64_t tiles = ((N + 255) / 256) * ((M + BM - 1) / BM);
  if (tiles >= 2 * 148 || K < 2048) return 1;
  auto fill = [](int64_t units) { return (double)units / (double)(((units + 147) / 148) * 148); };
  const int bn0 = tc_pick_bn(M, N, 0);
  const double eff0 = fill(((N + bn0 - 1) / bn0) * ((M + BM - 1) / BM));
  double best_eff = eff0 + 0.1;  // the extra workspace pass must buy a clear gain
  int64_t best = 1;
  for (int64_t S = 2; S <= 8 && K / S >= 1024; ++S) {
    const double eff = fill(tiles * S);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = S;
    }
  }
  if (best > 1) *bn_out = 256;
  return best;
}

int tc_gemm_prepare(TcGemm* g, const GemmShape& s, int epi, const EpiArgs& args, int bn_hint) {
  const int64_t M = s.M(), N = s.N(), K = s.K();
  if (M < 1 || N < 1 || K < 1 || s.KB() != K) return set_error(TTT_ERR_INVALID_ARG, "gemm: inconsistent shapes");
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return set_error(TTT_ERR_INVALID_ARG, "gemm: too large");
  if (epi < 0 || epi >= EPI_COUNT) return set_error(TTT_ERR_INVALID_ARG, "gemm: bad epilogue");
  const int bn = tc_pick_bn(M, N, bn_hint);
  if (epi == EPI_SWIGLU && (N % 128) != 0) return set_error(TTT_ERR_INVALID_ARG, "gemm: SwiGLU needs N % 128 == 0");
  if (bn == 160 && !(M > BM && pair_enabled() && (epi == EPI_STORE_F32 || epi == EPI_STORE_BF16 || epi == EPI_ADD_F32)))
    return set_error(TTT_ERR_INVALID_ARG, "gemm: 160-wide tiles need more than 128 rows and a store/add epilogue");
  g->a_mn = s.a_mn;
  g->b_mn = s.b_mn;
  g->bn = bn;
  g->epi = epi;
  g->M = M;
  g->N = N;
  g->K = K;
  g->args = args;
  g->ksplit = 1;
  g->kps = K;
  g->ws = nullptr;
  g->K2 = 0;
  g->n_ext = 0;
  g->pair = (M > BM && pair_enabled()) ? 1 : 0;
  int rc = make_tmap(&g->ta, s.a, s.a_mn ? 64 : BM);
  if (rc) return rc;
  rc = make_tmap(&g->tb, s.b, s.b_mn ? 64 : (g->pair ? bn / 2 : bn));
  g->ta2 = g->ta;
  g->tb2 = g->tb;
  return rc;
}

int tc_gemm_set_ext(TcGemm* g, const MatView& a2, const MatView& b2, int64_t n_ext) {
  const int64_t M2 = g->a_mn ? a2.cols : a2.rows, K2 = g->a_mn ? a2.rows : a2.cols;
  const int64_t N2 = g->b_mn ? b2.cols : b2.rows, KB = g->b_mn ? b2.rows : b2.cols;
  if (g->ksplit > 1) return set_error(TTT_ERR_STATE, "gemm: set the second product before split-K");
  if (K2 < 1 || KB != K2 || M2 != g->M || n_ext < 0 || n_ext % g->bn || N2 < g->N - n_ext)
    return set_error(TTT_ERR_INVALID_ARG, "gemm: inconsistent second product");
  if (g->epi == EPI_CE_FWD) return set_error(TTT_ERR_INVALID_ARG, "gemm: no second product with CE partials");
  int rc = make_tmap(&g->ta2, a2, g->a_mn ? 64 : BM);
  if (rc) return rc;
  rc = make_tmap(&g->tb2, b2, g->b_mn ? 64 : (g->pair ? g->bn / 2 : g->bn));
  if (rc) return rc;
  g->K2 = K2;
  g->n_ext = n_ext;
  return TTT_OK;
}

int tc_gemm_set_split(TcGemm* g, int64_t ksplit, float* ws) {
  if (ksplit <= 1) {
    g->ksplit = 1;
    g->kps = g->K;
    return TTT_OK;
  }
  if (!ws) return set_error(TTT_ERR_INVALID_ARG, "gemm: split-K needs a workspace");
  if (g->epi != EPI_STORE_F32 && g->epi != EPI_STORE_BF16 && g->epi != EPI_ADD_F32)
    return set_error(TTT_ERR_INVALID_ARG, "gemm: split-K only for store/add epilogues");
  if (g->K2 > 0 && g->n_ext > 0)
    return set_error(TTT_ERR_INVALID_ARG, "gemm: split-K needs the second product on every tile");
  // split the concatenated reduction in whole k-blocks
  const int64_t kblocks = (g->K + BK - 1) / BK + (g->K2 + BK - 1) / BK;
  const int64_t kpsb = (kblocks + ksplit - 1) / ksplit;
  g->ksplit = (int)((kblocks + kpsb - 1) / kpsb);
  g->kps = kpsb * BK;
  g->ws = ws;
  return TTT_OK;
}

int tc_gemm_launch(const TcGemm& g, cudaStream_t stream, int* dev_err) {
  const int kepi = g.ksplit > 1 ? EPI_STORE_F32 : g.epi;
  KernelFn fn = g.pair ? pick_pair(g.bn, g.a_mn, g.b_mn, kepi, g.act_bf16)
                       : (g.bn == 256 ? pick<256>(g.a_mn, g.b_mn, kepi, g.act_bf16)
                                      : pick<128>(g.a_mn, g.b_mn, kepi, g.act_bf16));
  if (!fn) return set_error(TTT_ERR_INVALID_ARG, "gemm: no kernel for this combination");
  const int smem = smem_bytes(g.pair, g.bn, kepi, g.b_mn);
  {
    static std::mutex mu;
    static std::set<std::pair<int, KernelFn>> configured;
    int dev = 0;
    TTT_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lock(mu);
    if (!configured.count({dev, fn})) {
      TTT_CUDA_TRY(cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
      configured.insert({dev, fn});
    }
  }
  // pairs: n_mt counts 256-row pair tiles and the grid is two CTAs per unit slot
  const int mrows = g.pair ? 2 * BM : BM;
  const int n_mt = (int)((g.M + mrows - 1) / mrows), n_nt = (int)((g.N + g.bn - 1) / g.bn);
  const int64_t units = (int64_t)n_mt * n_nt * g.ksplit;
  static int n_sm = 0;
  if (!n_sm) {
    int dev = 0;
    TTT_CUDA_TRY(cudaGetDevice(&dev));
    TTT_CUDA_TRY(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
  }
  int slots = n_sm;  // CTAs (or CTA pairs) that are resident at once
  if (g.pair) {
    // pairs that fit at the same time (a GPC with an odd number of free SMs
    // leaves one idle); a grid of more would run a second, partial wave
    static std::mutex mu;
    static std::map<std::pair<int, KernelFn>, int> pairs_of;
    int dev = 0;
    TTT_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lock(mu);
    auto it = pairs_of.find({dev, fn});
    if (it == pairs_of.end()) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2, 1, 1);
      cfg.blockDim = dim3(kGemmThreads, 1, 1);
      cfg.dynamicSmemBytes = (size_t)smem;
      int nc = 0;
      if (cudaOccupancyMaxActiveClusters(&nc, reinterpret_cast<const void*>(fn), &cfg) != cudaSuccess || nc < 1) {
        (void)cudaGetLastError();
        nc = n_sm / 2;
      }
      it = pairs_of.emplace(std::make_pair(dev, fn), std::min(nc, n_sm / 2)).first;
    }
    slots = it->second;
  }
  const dim3 grid(g.pair ? (unsigned)(2 * std::min<int64_t>(units, slots))
                         : (unsigned)std::min<int64_t>(units, slots));
  const int KB1 = (int)((g.K + BK - 1) / BK), KB2 = (int)((g.K2 + BK - 1) / BK);
  // n-tile fastest when B (N x K, plus a second product) fits comfortably in L2 and A is the larger
  // operand; when A and B are both larger than that, groups of m-tiles whose rows of A take about 24 MB
  const double a_bytes = 2.0 * (double)g.M * (double)(g.K + g.K2), b_bytes = 2.0 * (double)g.N * (double)(g.K + g.K2);
  int n_fast = (b_bytes <= 48e6 && a_bytes > b_bytes) ? 1 : 0;
  if (a_bytes > 48e6 && b_bytes > 48e6 && n_mt > 2) {
    const double tile_a = a_bytes / (double)n_mt;  // bytes of A per m-tile
    n_fast = (int)std::max(2.0, std::min(16.0, std::floor(24e6 / tile_a)));
  }
  const int64_t n_ext = g.K2 > 0 ? g.n_ext : INT64_MAX;
  if (g.ksplit <= 1) {
    fn<<<grid, kGemmThreads, smem, stream>>>(g.ta, g.tb, g.ta2, g.tb2, g.M, g.N, KB1, KB2, n_ext, KB1 + KB2, n_mt, n_nt, 1, n_fast,
                                    g.args, dev_err);
    TTT_CUDA_TRY(cudaGetLastError());
    return TTT_OK;
  }
  // split-K: partial accumulators to the workspace, then the ordered sum + epilogue
  EpiArgs part;
  part.c = g.ws;
  part.ldc = g.N;
  part.split_stride = g.M * g.N;
  fn<<<grid, kGemmThreads, smem, stream>>>(g.ta, g.tb, g.ta2, g.tb2, g.M, g.N, KB1, KB2, n_ext, (int)(g.kps / BK), n_mt, n_nt,
                                  g.ksplit, n_fast, part, dev_err);
  TTT_CUDA_TRY(cudaGetLastError());
  const unsigned blocks = ceil_div(g.M * ((g.N + 3) / 4), 256);
  switch (g.epi) {
    case EPI_STORE_F32:
      splitk_reduce_kernel<EPI_STORE_F32><<<blocks, 256, 0, stream>>>(g.ws, g.ksplit, g.M, g.N, g.M * g.N, g.args);
      break;
    case EPI_STORE_BF16:
      splitk_reduce_kernel<EPI_STORE_BF16><<<blocks, 256, 0, stream>>>(g.ws, g.ksplit, g.M, g.N, g.M * g.N, g.args);
      break;
    default:
      splitk_reduce_kernel<EPI_ADD_F32><<<blocks, 256, 0, stream>>>(g.ws, g.ksplit, g.M, g.N, g.M * g.N, g.args);
  }
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

}  // namespace ttt
