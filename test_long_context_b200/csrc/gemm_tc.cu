// Tensor-core GEMM for sm_100a: TMA tile loads into 128B-swizzled shared
// memory, tcgen05.mma (kind::f16, bf16 x bf16 -> fp32) issued by one thread,
// accumulator in TMEM, and a fused epilogue read back with tcgen05.ld.
//
// CTA = 6 warps: warp 0 lane 0 issues TMA, warp 1 owns the TMEM allocation
// and lane 0 issues the MMAs, warps 2..5 run the epilogue (warp w reads TMEM
// lanes 32*(w%4) .. +31, one accumulator row per thread).  Tile 128 x BN x 64,
// BN in {128, 256}, a 4- or 6-stage smem ring between producer and MMA.
#include <algorithm>
#include <mutex>
#include <set>

#include "gemm.cuh"
#include "ptx.cuh"

namespace ttt {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;

template <int BN>
struct TcCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int SMEM = STAGES * STAGE + 1024 /*align*/ + 256 /*barriers*/;
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
                                             const EpiArgs& ep, int tile_n) {
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
      if constexpr (EPI == EPI_STORE_F32) {
        store32<float>(reinterpret_cast<float*>(ep.c) + row * ep.ldc + col0, v, nval);
      } else if constexpr (EPI == EPI_STORE_BF16) {
        store32<bf16>(reinterpret_cast<bf16*>(ep.c) + row * ep.ldc + col0, v, nval);
      } else if constexpr (EPI == EPI_ADD_F32) {
        float* dst = reinterpret_cast<float*>(ep.c) + row * ep.ldc + col0;
        const float* src = ep.c2 ? reinterpret_cast<const float*>(ep.c2) + row * ep.ldc2 + col0 : dst;
        for (int i = 0; i < nval; ++i) v[i] += src[i];
        store32<float>(dst, v, nval);
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
      } else if constexpr (EPI == EPI_SGD) {
        float* w = reinterpret_cast<float*>(ep.c) + row * ep.ldc + col0;
        for (int i = 0; i < nval; ++i) v[i] = w[i] - ep.alpha * v[i];
        store32<float>(w, v, nval);
        if (ep.c2) store32<bf16>(reinterpret_cast<bf16*>(ep.c2) + row * ep.ldc2 + col0, v, nval);
      }
    }
  }
}

template <int BN, bool A_MN, bool B_MN, int EPI, typename TACT>
__global__ void __launch_bounds__(192, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb, int64_t M,
                   int64_t N, int64_t K, EpiArgs ep, int* err) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = (int64_t)blockIdx.x * BN, m0 = (int64_t)blockIdx.y * BM;
  const int nkb = (int)((K + BK - 1) / BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accf, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tma);
    ptx::prefetch_tmap(&tmb);
  }
  if (warp == 1) {
    __syncwarp();
    ptx::tmem_alloc(tmem_slot, BN);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % C::STAGES;
        const uint32_t ph = (uint32_t)(kb / C::STAGES) & 1u;
        if (!ptx::mbar_wait(&empty[s], ph ^ 1u, err)) break;
        ptx::mbar_arrive_expect_tx(&full[s], C::STAGE);
        uint8_t* a = sA + s * C::A_BYTES;
        uint8_t* b = sB + s * C::B_BYTES;
        const int k0 = kb * BK;
        if constexpr (!A_MN) {
          ptx::tma_load_2d(a, &tma, &full[s], k0, (int)m0);
        } else {
          ptx::tma_load_2d(a, &tma, &full[s], (int)m0, k0);
          ptx::tma_load_2d(a + 8192, &tma, &full[s], (int)m0 + 64, k0);
        }
        if constexpr (!B_MN) {
          ptx::tma_load_2d(b, &tmb, &full[s], k0, (int)n0);
        } else {
#pragma unroll
          for (int j = 0; j < BN / 64; ++j) ptx::tma_load_2d(b + j * 8192, &tmb, &full[s], (int)n0 + 64 * j, k0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(BM, BN, A_MN, B_MN);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % C::STAGES;
        const uint32_t ph = (uint32_t)(kb / C::STAGES) & 1u;
        if (!ptx::mbar_wait(&full[s], ph, err)) break;
        ptx::tc_fence_after();
        const uint32_t a_addr = ptx::smem_u32(sA + s * C::A_BYTES);
        const uint32_t b_addr = ptx::smem_u32(sB + s * C::B_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = A_MN ? ptx::smem_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                   : ptx::smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? ptx::smem_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                   : ptx::smem_desc_sw128(b_addr + kk * 32, 16, 1024);
          ptx::umma_bf16(tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        ptx::umma_commit(&empty[s]);
      }
      // Arrives once every MMA issued above has completed (also on a bail-out).
      ptx::umma_commit(accf);
      ptx::mbar_drain(accf, 0);  // no MMA may still write TMEM when it is released
    }
  } else {
    const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(accf, 0, err));  // warp-uniform before tcgen05.ld
    ptx::tc_fence_after();
    if (ok) {
      const int q = warp & 3;
      const int64_t row = m0 + q * 32 + lane;
      const uint32_t t_row = tmem + ((uint32_t)(q * 32) << 16);
      epilogue_row<BN, EPI, TACT>(t_row, row, row < M, n0, N, ep, (int)blockIdx.x);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();  // tcgen05.dealloc is warp-collective: reconverge lane 0 with the others
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, BN);
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

using KernelFn = void (*)(CUtensorMap, CUtensorMap, int64_t, int64_t, int64_t, EpiArgs, int*);

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

template <int BN>
KernelFn pick(int a_mn, int b_mn, int epi, int act_bf16) {
  if (!a_mn && !b_mn) return pick_epi<BN, false, false>(epi, act_bf16);
  if (!a_mn && b_mn) return pick_epi<BN, false, true>(epi, act_bf16);
  if (a_mn && b_mn) return pick_epi<BN, true, true>(epi, act_bf16);
  return pick_epi<BN, true, false>(epi, act_bf16);
}

}  // namespace

int64_t tc_ce_tiles(int64_t N, int bn) { return (N + bn - 1) / bn; }

int tc_pick_bn(int64_t M, int64_t N, int hint) {
  if (hint == 128 || hint == 256) return hint;
  // Prefer 256-wide tiles when that still gives every SM a tile.
  const int64_t tiles256 = ((N + 255) / 256) * ((M + BM - 1) / BM);
  return (tiles256 >= 148 || N > 4096) ? 256 : 128;
}

int tc_gemm_prepare(TcGemm* g, const GemmShape& s, int epi, const EpiArgs& args, int bn_hint) {
  const int64_t M = s.M(), N = s.N(), K = s.K();
  if (M < 1 || N < 1 || K < 1 || s.KB() != K) return set_error(TTT_ERR_INVALID_ARG, "gemm: inconsistent shapes");
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return set_error(TTT_ERR_INVALID_ARG, "gemm: too large");
  if (epi < 0 || epi >= EPI_COUNT) return set_error(TTT_ERR_INVALID_ARG, "gemm: bad epilogue");
  const int bn = tc_pick_bn(M, N, bn_hint);
  if (epi == EPI_SWIGLU && (N % 128) != 0) return set_error(TTT_ERR_INVALID_ARG, "gemm: SwiGLU needs N % 128 == 0");
  g->a_mn = s.a_mn;
  g->b_mn = s.b_mn;
  g->bn = bn;
  g->epi = epi;
  g->M = M;
  g->N = N;
  g->K = K;
  g->args = args;
  int rc = make_tmap(&g->ta, s.a, s.a_mn ? 64 : BM);
  if (rc) return rc;
  rc = make_tmap(&g->tb, s.b, s.b_mn ? 64 : bn);
  return rc;
}

int tc_gemm_launch(const TcGemm& g, cudaStream_t stream, int* dev_err) {
  KernelFn fn = g.bn == 256 ? pick<256>(g.a_mn, g.b_mn, g.epi, g.act_bf16) : pick<128>(g.a_mn, g.b_mn, g.epi, g.act_bf16);
  if (!fn) return set_error(TTT_ERR_INVALID_ARG, "gemm: no kernel for this combination");
  const int smem = g.bn == 256 ? TcCfg<256>::SMEM : TcCfg<128>::SMEM;
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
  dim3 grid((unsigned)((g.N + g.bn - 1) / g.bn), (unsigned)((g.M + BM - 1) / BM));
  fn<<<grid, 192, smem, stream>>>(g.ta, g.tb, g.M, g.N, g.K, g.args, dev_err);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

}  // namespace ttt
