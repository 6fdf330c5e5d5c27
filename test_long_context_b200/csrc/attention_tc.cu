// Tensor-core (tcgen05) flash attention forward for the banded causal window
// of eq. (1) (query p sees keys p-k+1 .. p), bf16 operands, fp32 softmax.
// Two forwards: the one below keeps a running row maximum and serves any
// inputs; the fixed-shift forward further down serves queries and keys of
// bounded norm (the model's QK-norm) and needs neither the maximum nor the
// rescaling of O.
//
// CTA = one tile of 128 queries x one head; 12 warps:
//   warp 0       TMA producer: Q once, then K/V tiles of 128 keys (2 stages)
//   warp 1       TMEM owner; lane 0 issues every tcgen05.mma
//   warps 4..11  softmax: two independent warpgroups; warpgroup g owns key
//                columns 64g..64g+63 of each tile and runs its own online
//                softmax into its own TMEM accumulator O_g (thread = query
//                row = TMEM lane), writes P (bf16) to 128B-swizzled smem and
//                rescales O_g only when its max grows by more than 2^8 (log2
//                domain); the epilogue combines O_0 and O_1 and writes O, LSE.
// S = Q K^T goes to one of two TMEM buffers (128 columns each) so that the
// next tile's QK^T overlaps this tile's softmax; O (head_dim columns) lives
// in TMEM for the whole key loop.
//
// head_dim = 64*A + R with R in {0, 16, 32}: the first 64*A columns of Q, K,
// V use 128-byte swizzled tiles, the remaining R columns a 2R-byte swizzle, so
// every TMA box starts on a 16-byte boundary and matches a canonical UMMA
// layout (K-major for Q and K, MN-major for V as the B operand of P V).
#include <mutex>
#include <set>

#include "attention_tc.cuh"
#include "ptx.cuh"

namespace ttt {
namespace {

constexpr int QT = 128;   // queries per CTA
constexpr int KT = 128;   // keys per tile
constexpr int NST = 2;    // K/V stages
constexpr float RESCALE_LOG2 = 8.f;

__host__ __device__ constexpr int rem_swizzle_layout(int rem) { return rem == 16 ? 6 : (rem == 32 ? 4 : 2); }

template <int HD>
struct Geo {
  static constexpr int A = HD / 64;          // 128B-swizzled atoms along head_dim
  static constexpr int R = HD % 64;          // remainder columns (0, 16, 32)
  static constexpr int RB = R * 2;           // remainder row bytes (32 or 64)
  static constexpr int TILE = 128 * HD * 2;  // bytes of a 128-row tile
  static constexpr int REM_OFF = A * 16384;  // offset of the remainder region in a tile
  // V tiles are whole 128B-swizzled atoms (the last one partly past the head),
  // so that one MMA of N = HD covers a P V step
  static constexpr int VA = (HD + 63) / 64;
  static constexpr int VTILE = VA * 16384;
  static constexpr int NK = HD <= 64 ? 4 : (HD <= 96 ? 3 : 2);  // K ring stages (released after S)
  static constexpr int NV = HD <= 64 ? 3 : 2;                    // V ring stages (released after P V)
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE;
  static constexpr int V_OFF = K_OFF + NK * TILE;
  static constexpr int P_OFF = V_OFF + NV * VTILE;
  static constexpr int P_BYTES = 128 * 128 * 2;
  static constexpr int BAR_OFF = P_OFF + 2 * P_BYTES;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static_assert(R == 0 || R == 16 || R == 32, "head_dim must be 64*A + {0,16,32}");
  static_assert(TILE % 1024 == 0, "tiles must stay 1024-byte aligned");
  static_assert(SMEM <= 232448, "shared memory per block");
};

__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)layout << 61;
  return d;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// AND of `v` over the `n` threads that meet at named barrier `id` (all of them
// must call it): lets a group agree on a bail-out before a later bar.sync.
__device__ __forceinline__ bool bar_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// 2^x with the hardware approximation (one MUFU op; -inf -> 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Paired fp32 arithmetic: one instruction for two values.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// 2^x for x <= 127 without the MUFU unit (x below -125 gives 2^-125).
// x = n + f with n the nearest integer (adding 1.5 * 2^23 rounds to it and
// leaves n in the low mantissa bits) and |f| <= 1/2; 2^f by a cubic whose
// coefficients are this library's own minimax fit of the relative error on
// [-1/2, 1/2] (Remez exchange; max relative error 7.5e-5, against bf16's 2^-9
// for P); 2^n is then added to the exponent field.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float2 sh = make_float2(12582912.f, 12582912.f);
  x = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
  const float2 t = fadd2(x, sh);
  const float2 f = fsub2(x, fsub2(t, sh));
  float2 p = ffma2(f, make_float2(0.0551716685f, 0.0551716685f), make_float2(0.242611125f, 0.242611125f));
  p = ffma2(p, f, make_float2(0.693260968f, 0.693260968f));
  p = ffma2(p, f, make_float2(0.999928057f, 0.999928057f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// P for W keys of one row under a fixed shift: p = 2^(s sl2 - m), packed as
// bf16 pairs (key 2i in the low half of pw[i]); returns the fp32 sum of p.
// Groups of 8 keys g with (g EMU) mod 8 < EMU use the polynomial, spread over
// the row so that MUFU and FMA work interleave; masked scores (-inf) need
// EMU = 0.
template <int EMU, int W>
__device__ __forceinline__ float emit_p_fixed(const float (&s)[W], float sl2, float neg_m, uint32_t (&pw)[W / 2]) {
  const float2 sc = make_float2(sl2, sl2), shift = make_float2(neg_m, neg_m);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int gr = 0; gr < W / 8; ++gr) {
    const bool poly = ((gr * EMU) & 7) < EMU;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = gr * 8 + 2 * i;
      const float2 x = ffma2(make_float2(s[c], s[c + 1]), sc, shift);
      const float2 e = poly ? exp2_poly2(x) : make_float2(ex2(x.x), ex2(x.y));
      if (i & 1)
        acc1 = fadd2(acc1, e);
      else
        acc0 = fadd2(acc0, e);
      __nv_bfloat162 b = __floats2bfloat162_rn(e.x, e.y);
      pw[c / 2] = *reinterpret_cast<uint32_t*>(&b);
    }
  }
  const float2 t = fadd2(acc0, acc1);
  return t.x + t.y;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Load one 128-row tile (rows row0.., head columns col0 .. col0+HD) into smem.
template <int HD>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* m128, const CUtensorMap* mrem,
                                          uint64_t* bar, int col0, int row0) {
  using G = Geo<HD>;
#pragma unroll
  for (int a = 0; a < G::A; ++a) ptx::tma_load_2d(dst + a * 16384, m128, bar, col0 + 64 * a, row0);
  if constexpr (G::R > 0) ptx::tma_load_2d(dst + G::REM_OFF, mrem, bar, col0 + 64 * G::A, row0);
}

template <int HD>
__global__ void __launch_bounds__(384, 1)
    swa_fwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tq_r,
                      const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tk_r,
                      const __grid_constant__ CUtensorMap tv, SwaArgs a, int* err) {
  using G = Geo<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + G::BAR_OFF);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;              // [NK]
  uint64_t* k_empty = k_full + G::NK;       // [NK]
  uint64_t* v_full = k_empty + G::NK;       // [NV]
  uint64_t* v_empty = v_full + G::NV;       // [NV]
  uint64_t* s_full = v_empty + G::NV;       // [2]
  uint64_t* s_empty = s_full + 2;           // [2]
  uint64_t* p_full = s_empty + 2;           // [2]
  uint64_t* pv_done = p_full + 2;           // [2]
  uint64_t* o_full = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_full + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t q0 = a.p0 + (int64_t)blockIdx.x * QT;            // absolute position of row 0
  const int64_t qlast = imin64(q0 + QT, a.p0 + a.n) - 1;          // last valid query position
  const int64_t kfirst = imax64(0, q0 - a.window + 1);
  const int64_t j_begin = (kfirst / KT) * KT;                     // aligned key tile start
  const int ntiles = (int)((qlast - j_begin) / KT + 1);
  const int col0 = h * HD;

  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 1);
    for (int s = 0; s < G::NK; ++s) {
      ptx::mbar_init(&k_full[s], 1);
      ptx::mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < G::NV; ++s) {
      ptx::mbar_init(&v_full[s], 1);
      ptx::mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&s_full[s], 1);
      ptx::mbar_init(&s_empty[s], 256);
      ptx::mbar_init(&p_full[s], 256);
      ptx::mbar_init(&pv_done[s], 1);
    }
    ptx::mbar_init(o_full, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // S buffers at columns 0 and 128; O_0, O_1 (one per key half / softmax warpgroup) at 256 and 384
  const uint32_t t_s0 = tmem, t_o0 = tmem + 256, t_o1 = tmem + 384;

  if (warp == 0) {
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(q_full, G::TILE);
      load_tile<HD>(sm + G::Q_OFF, &tq, &tq_r, q_full, col0, (int)(q0 - a.p0));
      // K runs one tile ahead of V: K_{j+1} is wanted for S_{j+1} before P_j V_j
      auto load_k = [&](int j) {
        const int s = j % G::NK;
        if (!ptx::mbar_wait(&k_empty[s], ((j / G::NK) & 1) ^ 1, err)) return false;
        ptx::mbar_arrive_expect_tx(&k_full[s], G::TILE);
        const int slot = (int)((j_begin + (int64_t)j * KT) % a.ring);
        load_tile<HD>(sm + G::K_OFF + s * G::TILE, &tk, &tk_r, &k_full[s], col0, slot);
        return true;
      };
      bool ok = ntiles > 0 ? load_k(0) : true;
      for (int j = 0; ok && j < ntiles; ++j) {
        if (j + 1 < ntiles && !(ok = load_k(j + 1))) break;
        const int s = j % G::NV;
        if (!(ok = ptx::mbar_wait(&v_empty[s], ((j / G::NV) & 1) ^ 1, err))) break;
        ptx::mbar_arrive_expect_tx(&v_full[s], G::VTILE);
        const int slot = (int)((j_begin + (int64_t)j * KT) % a.ring);
        uint8_t* vd = sm + G::V_OFF + s * G::VTILE;
#pragma unroll
        for (int at = 0; at < G::VA; ++at) ptx::tma_load_2d(vd + at * 16384, &tv, &v_full[s], col0 + 64 * at, slot);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_s = ptx::idesc_bf16_f32(128, KT, false, false);
      constexpr uint32_t id_pv = ptx::idesc_bf16_f32(128, HD, false, true);
      const uint32_t q_addr = ptx::smem_u32(sm + G::Q_OFF);
      bool ok = ptx::mbar_wait(q_full, 0, err);
      auto issue_s = [&](int j) {
        const int s = j % G::NK;
        const uint32_t k_addr = ptx::smem_u32(sm + G::K_OFF + s * G::TILE);
        const uint32_t d = t_s0 + (j & 1) * 128;
        int step = 0;
#pragma unroll
        for (int at = 0; at < G::A; ++at)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk, ++step)
            ptx::umma_bf16(d, sdesc(q_addr + at * 16384 + kk * 32, 16, 1024, 2),
                           sdesc(k_addr + at * 16384 + kk * 32, 16, 1024, 2), id_s, step > 0);
        if constexpr (G::R > 0) {
#pragma unroll
          for (int kk = 0; kk < G::R / 16; ++kk, ++step)
            ptx::umma_bf16(d, sdesc(q_addr + G::REM_OFF + kk * 32, 16, 8 * G::RB, rem_swizzle_layout(G::R)),
                           sdesc(k_addr + G::REM_OFF + kk * 32, 16, 8 * G::RB, rem_swizzle_layout(G::R)), id_s,
                           step > 0);
        }
        ptx::umma_commit(&s_full[j & 1]);
        ptx::umma_commit(&k_empty[s]);
      };
      if (ok && ntiles > 0) {
        if ((ok = ptx::mbar_wait(&k_full[0], 0, err))) {
          ptx::tc_fence_after();
          issue_s(0);
        }
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        if (j + 1 < ntiles) {
          const int s1 = (j + 1) % G::NK;
          if (!(ok = ptx::mbar_wait(&k_full[s1], ((j + 1) / G::NK) & 1, err))) break;
          if (j + 1 >= 2 && !(ok = ptx::mbar_wait(&s_empty[(j + 1) & 1], (((j + 1) / 2) - 1) & 1, err))) break;
          ptx::tc_fence_after();
          issue_s(j + 1);
        }
        const int sv = j % G::NV;
        if (!(ok = ptx::mbar_wait(&p_full[j & 1], (j / 2) & 1, err))) break;
        if (!(ok = ptx::mbar_wait(&v_full[sv], (j / G::NV) & 1, err))) break;
        ptx::tc_fence_after();
        const uint32_t v_addr = ptx::smem_u32(sm + G::V_OFF + sv * G::VTILE);
        const uint32_t p_addr = ptx::smem_u32(sm + G::P_OFF + (j & 1) * G::P_BYTES);
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {  // keys 0..63 -> O_0, keys 64..127 -> O_1
          const uint64_t pd = sdesc(p_addr + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024, 2);
          const uint32_t acc = (j > 0 || (kk % 4) > 0) ? 1u : 0u;
          // V: MN-major, VA atoms 16384 bytes apart along head_dim (LBO), 8-key groups 1024 apart (SBO)
          ptx::umma_bf16(kk < 4 ? t_o0 : t_o1, pd, sdesc(v_addr + kk * 2048, 16384, 1024, 2), id_pv, acc);
        }
        ptx::umma_commit(&v_empty[sv]);
        ptx::umma_commit(&pv_done[j & 1]);
      }
      ptx::umma_commit(o_full);
      ptx::mbar_drain(o_full, 0);  // no MMA may still write TMEM when it is released
    }
  } else if (warp >= 4) {
    // ---- softmax: two independent warpgroups.  Warpgroup g owns key columns
    // 64g .. 64g+63 of every tile and runs its own online softmax (max m, sum l)
    // into its own accumulator O_g; thread = query row (= TMEM lane).  The two
    // halves are combined once, in the epilogue. ----
    const int g = (warp - 4) >> 2;
    const int r = ((warp - 4) & 3) * 32 + lane;
    const int64_t p = q0 + r;
    const bool row_ok = p <= qlast;
    const uint32_t lane_off = (uint32_t)(((warp - 4) & 3) * 32) << 16;
    const uint32_t t_og = g ? t_o1 : t_o0;
    const float sl2 = a.scale * 1.4426950408889634f;        // scale * log2(e)
    // epilogue exchange of the halves' row statistics, in P buffer 0 (free once O is final)
    float* xm = reinterpret_cast<float*>(sm + G::P_OFF);  // [2][128] row max per half
    float* xl = xm + 256;                                 // [2][128] row sum per half
    float m = -INFINITY, l = 0.f;
    uint8_t* pbase = sm + G::P_OFF;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int64_t j0 = j_begin + (int64_t)j * KT + 64 * g;  // position of this half's first key
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s_full[j & 1], (j / 2) & 1, err));
      if (!ok) break;  // warp-uniform: TMEM loads follow
      ptx::tc_fence_after();
      float s[64];  // raw scores; the scale is folded into the exponent
      {
        uint32_t rr[64];  // one TMEM round trip for the warp's 64 columns
        ptx::tmem_ld64(t_s0 + (j & 1) * 128 + 64 * g + lane_off, rr);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 64; ++i) s[i] = __uint_as_float(rr[i]);
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&s_empty[j & 1]);
      const int64_t lo = p - a.window + 1 - j0, hi = p - j0;  // key c valid iff lo <= c <= hi
      if (!(row_ok && lo <= 0 && hi >= 63)) {
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = (row_ok && c >= lo && c <= hi) ? s[c] : -INFINITY;
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) mx[u] = fmaxf(mx[u], s[c + u]);
      }
      const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;  // log2 domain
      // lazy rescaling of O_g (needs PV_{j-1} complete); warp-collective TMEM
      // access, so a warp rescales together when any of its rows needs it
      float mu = m, corr = 1.f;
      if (tmax > -INFINITY) {
        if (m == -INFINITY) {
          mu = tmax;
        } else if (tmax > m + RESCALE_LOG2) {
          mu = tmax;
          corr = ex2(m - mu);
          l *= corr;
        }
      }
      m = mu;
      if (__any_sync(0xffffffffu, corr != 1.f)) {
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) / 2) & 1, err));
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int c = 0; c < HD; c += 16) {
          uint32_t o[16];
          tmem_ld16(t_og + c + lane_off, o);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
          tmem_st16(t_og + c + lane_off, o);
        }
        tmem_st_wait();
      }
      if (j >= 2) {  // P buffer (j & 1) is free once PV_{j-2} completed
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&pv_done[j & 1], ((j - 2) / 2) & 1, err));
        if (!ok) break;
      }
      uint8_t* prow = pbase + (j & 1) * G::P_BYTES + g * 16384 + r * 128;  // this half = one 64-key atom
      const float neg_m = (m == -INFINITY) ? 0.f : -m;  // m = -inf only while every score so far is masked
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int gr = 0; gr < 8; ++gr) {  // 8 granules of 8 keys
        float pv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          pv[i] = ex2(fmaf(s[gr * 8 + i], sl2, neg_m));
          ls[i & 3] += pv[i];
        }
        uint4 w;
        __nv_bfloat162 b0 = __floats2bfloat162_rn(pv[0], pv[1]), b1 = __floats2bfloat162_rn(pv[2], pv[3]);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(pv[4], pv[5]), b3 = __floats2bfloat162_rn(pv[6], pv[7]);
        w.x = *reinterpret_cast<uint32_t*>(&b0);
        w.y = *reinterpret_cast<uint32_t*>(&b1);
        w.z = *reinterpret_cast<uint32_t*>(&b2);
        w.w = *reinterpret_cast<uint32_t*>(&b3);
        *reinterpret_cast<uint4*>(prow + ((gr ^ (r & 7)) << 4)) = w;
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&p_full[j & 1]);
    }
    // ---- epilogue: combine the halves, O = (O_0 2^(m_0-M) + O_1 2^(m_1-M)) / l ----
    if (ok) ok = ptx::mbar_wait(o_full, 0, err);
    ok = bar_and(1, 256, ok);  // every softmax thread arrives here exactly once
    if (ok) {
      xm[g * 128 + r] = m;
      xl[g * 128 + r] = l;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      const float m0 = xm[r], m1 = xm[128 + r];
      const float M = fmaxf(m0, m1);
      const float f0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M), f1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M);
      const float lt = xl[r] * f0 + xl[128 + r] * f1;
      ptx::tc_fence_after();
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float c0 = f0 * inv, c1 = f1 * inv;
      const int64_t i = p - a.p0;
      bf16* orow = reinterpret_cast<bf16*>(a.o) + i * a.ldo + col0;
#pragma unroll
      for (int c = 16 * g; c < HD; c += 32) {  // this thread writes the 16-column groups of parity g
        uint32_t o0[16], o1[16];
        tmem_ld16(t_o0 + c + lane_off, o0);
        tmem_ld16(t_o1 + c + lane_off, o1);
        ptx::tmem_ld_wait();
        if (row_ok) {
          uint32_t pw[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float v0 = __uint_as_float(o0[2 * e]) * c0 + __uint_as_float(o1[2 * e]) * c1;
            const float v1 = __uint_as_float(o0[2 * e + 1]) * c0 + __uint_as_float(o1[2 * e + 1]) * c1;
            __nv_bfloat162 t2 = __floats2bfloat162_rn(v0, v1);
            pw[e] = *reinterpret_cast<uint32_t*>(&t2);
          }
          *reinterpret_cast<uint4*>(orow + c) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
          *reinterpret_cast<uint4*>(orow + c + 8) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
        }
      }
      if (row_ok && g == 0) a.lse[(int64_t)h * a.ld_lse + i] = (M + log2f(lt)) * 0.6931471805599453f;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();  // tcgen05.dealloc is warp-collective: reconverge lane 0 with the others
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// Forward with a fixed softmax shift, for query and key rows of bounded norm
// (|q| <= qmax, |k| <= kmax, as after the model's QK-norm).  Cauchy-Schwarz
// bounds every score of query row r: q_r.k <= |q_r| kmax, and softmax is
// invariant to a per-row shift, so each row exponentiates
// 2^(s scale log2e - m_r) with m_r = scale log2e |q_r| kmax (1% above, for
// the bf16 rounding of the keys) instead of a running maximum: no max
// reduction, no rescaling of O, one O accumulator for every key.  The host
// takes this kernel only when scale log2e qmax kmax <= 48, so the largest
// term of a row is >= 2^-96 and terms 2^30 below it are still normal floats.
//
// CTA = 128 queries x one head; key tiles of 128 keys; 4 + 4 NWG warps:
//   warp 0      TMA producer: K_j and V_j into stage j % NS (both released
//               by the MMAs that read them)
//   warp 1      TMEM owner; lane 0 issues S_j = Q K_j^T into S buffer j & 1
//               (Q read from TMEM) two tiles ahead, and O += P_j V_j once P_j
//               is in TMEM (A operand read from TMEM, over S_j's own columns)
//   warps 4..   NWG softmax warpgroups; warpgroup g owns key columns
//               [g W, g W + W) of every tile, W = 128 / NWG; thread = query
//               row = TMEM lane.  Each first writes its part of its row of Q
//               into TMEM (bf16 pairs), then per tile: S from TMEM, P =
//               2^(...) with part of the exponentials (EMU of every 8 groups
//               of 8 keys) from an FMA-pipe polynomial instead of the MUFU
//               unit, and bf16 P written back over the first W/2 columns of
//               its own S columns.
// Only the K and V tiles go through shared memory: the tensor core reads Q
// and P from TMEM, so shared-memory bandwidth serves the TMA writes and the B
// operands alone.
// TMEM: S/P buffers at columns 0 and 128, O at 256 (head_dim columns), Q at
// 384 (head_dim / 2 columns of bf16 pairs).
template <int HD>
struct FxGeo {
  static constexpr int A = HD / 64;
  static constexpr int R = HD % 64;
  static constexpr int KTILE = 128 * HD * 2;  // A 128B-swizzled atoms + the remainder box
  static constexpr int REM_OFF = A * 16384;
  static constexpr int VA = (HD + 63) / 64;
  static constexpr int VTILE = VA * 16384;  // whole atoms: one MMA of N = HD per 16 keys
  static constexpr int NS = HD == 64 ? 6 : (HD == 80 ? 4 : 3);
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = NS * KTILE;
  static constexpr int X_OFF = V_OFF + NS * VTILE;  // [4][128] fp32 row sums of the warpgroups
  static constexpr int BAR_OFF = X_OFF + 4 * 128 * 4;
  static constexpr int SMEM = BAR_OFF + 512 + 1024;
  static_assert(KTILE % 1024 == 0 && VTILE % 1024 == 0, "1024-byte aligned stages");
  static_assert(SMEM <= 232448, "shared memory per block");
  static_assert(HD / 2 <= 128, "Q columns");
};

template <int HD, int EMU, int NWG>
__global__ void __launch_bounds__(128 + 128 * NWG, 1)
    swa_fwd_fx_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tk_r,
                      const __grid_constant__ CUtensorMap tv, SwaArgs a, int* err) {
  using G = FxGeo<HD>;
  constexpr int W = 128 / NWG;     // key columns per softmax warpgroup
  constexpr int NSM = 128 * NWG;   // softmax threads
  constexpr int NS = G::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + G::BAR_OFF);
  uint64_t* k_full = bars;            // [NS]
  uint64_t* k_empty = k_full + NS;    // [NS]
  uint64_t* v_full = k_empty + NS;    // [NS]
  uint64_t* v_empty = v_full + NS;    // [NS]
  uint64_t* s_full = v_empty + NS;    // [2]  S_j in TMEM buffer j & 1
  uint64_t* s_free = s_full + 2;      // [2]  PV_j done: buffer j & 1 may take S_{j+2}
  uint64_t* p_full = s_free + 2;      // [2]  P_j written over S_j
  uint64_t* q_full = p_full + 2;      // Q in TMEM
  uint64_t* o_full = q_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_full + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t q0 = a.p0 + (int64_t)blockIdx.x * QT;
  const int64_t qlast = imin64(q0 + QT, a.p0 + a.n) - 1;
  const int64_t kfirst = imax64(0, q0 - a.window + 1);
  const int64_t j_begin = (kfirst / KT) * KT;
  const int ntiles = (int)((qlast - j_begin) / KT + 1);
  const int col0 = h * HD;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(&k_full[s], 1);
      ptx::mbar_init(&k_empty[s], 1);
      ptx::mbar_init(&v_full[s], 1);
      ptx::mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&s_full[s], 1);
      ptx::mbar_init(&s_free[s], 1);
      ptx::mbar_init(&p_full[s], NSM);
    }
    ptx::mbar_init(q_full, NSM);
    ptx::mbar_init(o_full, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s = tmem, t_o = tmem + 256, t_q = tmem + 384;

  if (warp == 0) {
    {  // the converged warp polls the rings; lane 0 issues the loads
      bool ok = true;
      for (int j = 0; ok && j < ntiles; ++j) {
        const int s = j % NS;
        const uint32_t ph = ((j / NS) & 1) ^ 1;
        const int slot = (int)((j_begin + (int64_t)j * KT) % a.ring);
        if (!(ok = ptx::mbar_wait_warp(&k_empty[s], ph, err))) break;
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(&k_full[s], G::KTILE);
          load_tile<HD>(sm + G::K_OFF + s * G::KTILE, &tk, &tk_r, &k_full[s], col0, slot);
        }
        if (!(ok = ptx::mbar_wait_warp(&v_empty[s], ph, err))) break;
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(&v_full[s], G::VTILE);
          uint8_t* vd = sm + G::V_OFF + s * G::VTILE;
#pragma unroll
          for (int at = 0; at < G::VA; ++at)
            ptx::tma_load_2d(vd + at * 16384, &tv, &v_full[s], col0 + 64 * at, slot);
        }
      }
    }
  } else if (warp == 1) {
    {  // the converged warp runs the issue loop; one elected lane issues each MMA and commit
      constexpr uint32_t id_s = ptx::idesc_bf16_f32(128, KT, false, false);
      constexpr uint32_t id_pv = ptx::idesc_bf16_f32(128, HD, false, true);
      bool ok = ptx::mbar_wait_warp(q_full, 0, err);
      auto issue_s = [&](int j) {
        const int s = j % NS;
        if (!ptx::mbar_wait_warp(&k_full[s], (j / NS) & 1, err)) return false;
        if (j >= 2 && !ptx::mbar_wait_warp(&s_free[j & 1], ((j - 2) / 2) & 1, err)) return false;
        ptx::tc_fence_after();
        const uint32_t k_addr = ptx::smem_u32(sm + G::K_OFF + s * G::KTILE);
        const uint32_t d = t_s + (j & 1) * 128;
        int step = 0;
#pragma unroll
        for (int at = 0; at < G::A; ++at)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk, ++step)
            ptx::umma_bf16_ts_elect(d, t_q + (at * 64 + kk * 16) / 2, sdesc(k_addr + at * 16384 + kk * 32, 16, 1024, 2),
                              id_s, step > 0);
        if constexpr (G::R > 0) {
#pragma unroll
          for (int kk = 0; kk < G::R / 16; ++kk, ++step)
            ptx::umma_bf16_ts_elect(d, t_q + (G::A * 64 + kk * 16) / 2,
                              sdesc(k_addr + G::REM_OFF + kk * 32, 16, 8 * G::R * 2, rem_swizzle_layout(G::R)), id_s,
                              step > 0);
        }
        ptx::umma_commit_elect(&s_full[j & 1]);
        ptx::umma_commit_elect(&k_empty[s]);
        return true;
      };
      if (ok && ntiles > 0) ok = issue_s(0);
      if (ok && ntiles > 1) ok = issue_s(1);
      for (int j = 0; ok && j < ntiles; ++j) {
        const int s = j % NS;
        if (!(ok = ptx::mbar_wait_warp(&p_full[j & 1], (j / 2) & 1, err))) break;
        if (!(ok = ptx::mbar_wait_warp(&v_full[s], (j / NS) & 1, err))) break;
        ptx::tc_fence_after();
        const uint32_t v_addr = ptx::smem_u32(sm + G::V_OFF + s * G::VTILE);
        const uint32_t pbuf = t_s + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {  // keys 16 kk .. 16 kk + 15: warpgroup gk's P columns
          const int gk = (kk * 16) / W;
          const uint32_t pa = pbuf + gk * W + (kk * 16 - gk * W) / 2;
          // V: MN-major, VA atoms 16384 bytes apart along head_dim (LBO), 8-key groups 1024 apart (SBO)
          ptx::umma_bf16_ts_elect(t_o, pa, sdesc(v_addr + kk * 2048, 16384, 1024, 2), id_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::umma_commit_elect(&v_empty[s]);
        ptx::umma_commit_elect(&s_free[j & 1]);
        if (j + 2 < ntiles && !(ok = issue_s(j + 2))) break;
      }
      ptx::umma_commit_elect(o_full);
      ptx::mbar_drain(o_full, 0);  // no MMA may still write TMEM when it is released
    }
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;
    const int quarter = warp & 3;  // TMEM lane quarter
    const int r = quarter * 32 + lane;
    const int64_t p = q0 + r;
    const bool row_ok = p <= qlast;
    const int64_t i = p - a.p0;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = a.scale * 1.4426950408889634f;
    // this warpgroup's 8-column groups of the row of Q (bf16 pairs) into TMEM; |q_r|^2 over all of it
    float qq = 0.f;
    {
      const bf16* src = reinterpret_cast<const bf16*>(a.q) + i * a.ldq + col0;
#pragma unroll
      for (int c8 = 0; c8 < HD / 16; ++c8) {
        uint4 u0 = make_uint4(0u, 0u, 0u, 0u), u1 = u0;
        if (row_ok) {
          u0 = *reinterpret_cast<const uint4*>(src + 16 * c8);
          u1 = *reinterpret_cast<const uint4*>(src + 16 * c8 + 8);
        }
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
          qq = fmaf(f2.x, f2.x, fmaf(f2.y, f2.y, qq));
        }
        if (c8 % NWG == g) ptx::tmem_st8(t_q + lane_off + 8 * c8, w);
      }
      tmem_st_wait();
      ptx::tc_fence_before();
      ptx::mbar_arrive(q_full);
    }
    const float m_fix = sqrtf(qq) * a.k_norm_max * sl2 * 1.01f;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int64_t j0 = j_begin + (int64_t)j * KT + g * W;  // position of this warpgroup's first key
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s_full[j & 1], (j / 2) & 1, err));
      if (!ok) break;  // warp-uniform: TMEM accesses follow
      ptx::tc_fence_after();
      const uint32_t tcol = t_s + (j & 1) * 128 + g * W + lane_off;
      float s[W];
      {
        uint32_t rr[W];
        if constexpr (W == 64)
          ptx::tmem_ld64(tcol, rr);
        else
          ptx::tmem_ld32(tcol, rr);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < W; ++c) s[c] = __uint_as_float(rr[c]);
      }
      const int64_t lo = p - a.window + 1 - j0, hi = p - j0;  // key c valid iff lo <= c <= hi
      const bool full = row_ok && lo <= 0 && hi >= W - 1;
      if (!full) {
#pragma unroll
        for (int c = 0; c < W; ++c) s[c] = (row_ok && c >= lo && c <= hi) ? s[c] : -INFINITY;
      }
      uint32_t pw[W / 2];
      l += __all_sync(0xffffffffu, full) ? emit_p_fixed<EMU, W>(s, sl2, -m_fix, pw)
                                         : emit_p_fixed<0, W>(s, sl2, -m_fix, pw);
      if constexpr (W == 64)
        tmem_st32(tcol, pw);
      else
        tmem_st16(tcol, pw);
      tmem_st_wait();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&p_full[j & 1]);
    }
    // ---- epilogue: O / l, l summed over the warpgroups ----
    if (ok) ok = ptx::mbar_wait(o_full, 0, err);
    ok = bar_and(1, NSM, ok);  // every softmax thread arrives here exactly once
    if (ok) {
      float* xl = reinterpret_cast<float*>(sm + G::X_OFF);
      xl[g * 128 + r] = l;
      asm volatile("bar.sync 1, %0;" ::"r"(NSM) : "memory");
      float lt = 0.f;
#pragma unroll
      for (int w = 0; w < NWG; ++w) lt += xl[w * 128 + r];
      ptx::tc_fence_after();
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      bf16* orow = reinterpret_cast<bf16*>(a.o) + i * a.ldo + col0;
#pragma unroll
      for (int c = 16 * g; c < HD; c += 16 * NWG) {  // this warpgroup's 16-column groups
        uint32_t o[16];
        tmem_ld16(t_o + c + lane_off, o);
        ptx::tmem_ld_wait();
        if (row_ok) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            __nv_bfloat162 t2 = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
            pk[e] = *reinterpret_cast<uint32_t*>(&t2);
          }
          *reinterpret_cast<uint4*>(orow + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(orow + c + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      if (row_ok && g == 0) a.lse[(int64_t)h * a.ld_lse + i] = (m_fix + log2f(lt)) * 0.6931471805599453f;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();  // tcgen05.dealloc is warp-collective: reconverge lane 0 with the others
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

template <int HD>
__device__ __forceinline__ void load_rows(uint8_t* dst, const CUtensorMap* m64, const CUtensorMap* mrem,
                                          uint64_t* bar, int col0, int row0, int atom_bytes, int rem_off) {
  constexpr int A = HD / 64, R = HD % 64;
#pragma unroll
  for (int a = 0; a < A; ++a) ptx::tma_load_2d(dst + a * atom_bytes, m64, bar, col0 + 64 * a, row0);
  if constexpr (R > 0) ptx::tma_load_2d(dst + rem_off, mrem, bar, col0 + 64 * A, row0);
}

// ---------------------------------------------------------------------------------------------
// Backward, dq part: dQ = scale * sum_j dS_j K_j over the band, with
// dS = P o (dP - D), P = exp(S*scale - lse), S = Q K^T, dP = dO V^T; the
// softmax statistics come from the forward (lse), so the tiles of a row are
// independent.  Tiles of 128 keys: 18 MMAs per 128 keys (S and dP of
// N = 128, then dQ += dS K as 8 MMAs of N = head_dim) where 64-key tiles
// need 28, and a single-CTA MMA costs about 100 cycles whatever its N.
// CTA = 128 queries x one head; 12 warps:
//   warp 0      TMA: K tiles (ring of NK, released after dQ_j) and V tiles
//               (ring of NV, released after dP_j), 128 keys as whole
//               128B-swizzled atoms; one lane per atom
//   warp 1      TMEM owner; the converged warp issues S_j = Q K_j^T and
//               dP_j = dO V_j^T (A operands Q and dO from TMEM) into one TMEM
//               buffer, then dQ += dS_j K_j once both warpgroups wrote dS_j
//   warps 4..11 two warpgroups owning key columns 64g .. 64g+63 of every tile:
//               thread = query row; P = 2^(S scale log2e - lse log2e),
//               dS = P o (dP - D) -> bf16 into the 128B-swizzled dS tile (one
//               64-key atom per warpgroup, double-buffered)
// TMEM: S at columns 0..127, dP at 128..255, dQ at 256, Q and dO (bf16 pairs)
// from 384.  S and dP of tile j+1 are issued as soon as both warpgroups have
// read tile j's, so they run under tile j's dS arithmetic.
constexpr int DKT = 128;

template <int HD>
struct DGeo {
  static constexpr int KA = (HD + 63) / 64;         // whole atoms of a K or V tile
  static constexpr int KTILE = DKT * 128 * KA;      // 128 keys x KA atoms of 128 B per row
  static constexpr int NK = KA == 1 ? 4 : 3;        // K stages (released after dQ_j)
  static constexpr int NV = KA == 1 ? 3 : 2;        // V stages (released after dP_j)
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + NK * KTILE;
  static constexpr int DS_OFF = V_OFF + NV * KTILE;
  static constexpr int DS_BYTES = 128 * DKT * 2;    // two 64-key atoms
  static constexpr int BAR_OFF = DS_OFF + 2 * DS_BYTES;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static_assert(KTILE % 1024 == 0, "1024-byte aligned tiles");
  static_assert(SMEM <= 232448, "shared memory per block");
};

template <int HD>
__global__ void __launch_bounds__(384, 1)
    swa_bwd_dq128_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv, SwaArgs a,
                         int* err) {
  using G = DGeo<HD>;
  constexpr int NK = G::NK, NV = G::NV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + G::BAR_OFF);
  uint64_t* q_full = bars + 0;        // Q and dO written to TMEM
  uint64_t* k_full = bars + 1;        // [NK]
  uint64_t* k_empty = k_full + NK;    // [NK]
  uint64_t* v_full = k_empty + NK;    // [NV]
  uint64_t* v_empty = v_full + NV;    // [NV]
  uint64_t* s_full = v_empty + NV;    // S_j and dP_j in TMEM
  uint64_t* s_empty = s_full + 1;     // both warpgroups read S_j and dP_j
  uint64_t* ds_full = s_empty + 1;    // [2] dS_j written
  uint64_t* ds_free = ds_full + 2;    // [2] dQ_j consumed dS buffer j&1
  uint64_t* dq_full = ds_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dq_full + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t q0 = a.p0 + (int64_t)blockIdx.x * QT;
  const int64_t qlast = imin64(q0 + QT, a.p0 + a.n) - 1;
  const int64_t kfirst = imax64(0, q0 - a.window + 1);
  const int64_t j_begin = (kfirst / DKT) * DKT;
  const int ntiles = (int)((qlast - j_begin) / DKT + 1);
  const int col0 = h * HD;

  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 256);
    for (int s = 0; s < NK; ++s) {
      ptx::mbar_init(&k_full[s], 1);
      ptx::mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      ptx::mbar_init(&v_full[s], 1);
      ptx::mbar_init(&v_empty[s], 1);
    }
    ptx::mbar_init(s_full, 1);
    ptx::mbar_init(s_empty, 256);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&ds_full[s], 256);
      ptx::mbar_init(&ds_free[s], 1);
    }
    ptx::mbar_init(dq_full, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s = tmem, t_dp = tmem + 128, t_dq = tmem + 256, t_q = tmem + 384, t_do = t_q + HD / 2;

  if (warp == 0) {
    {  // the converged warp polls the rings; one lane per atom issues the loads
      bool ok = true;
      for (int j = 0; ok && j < ntiles; ++j) {
        const int slot = (int)((j_begin + (int64_t)j * DKT) % a.ring);
        const int sk = j % NK, sv = j % NV;
        if (!(ok = ptx::mbar_wait_warp(&k_empty[sk], ((j / NK) & 1) ^ 1, err))) break;
        if (lane == 0) ptx::mbar_arrive_expect_tx(&k_full[sk], G::KTILE);
        __syncwarp();
        if (lane < G::KA)
          ptx::tma_load_2d(sm + G::K_OFF + sk * G::KTILE + lane * 16384, &tk, &k_full[sk], col0 + 64 * lane, slot);
        if (!(ok = ptx::mbar_wait_warp(&v_empty[sv], ((j / NV) & 1) ^ 1, err))) break;
        if (lane == 0) ptx::mbar_arrive_expect_tx(&v_full[sv], G::KTILE);
        __syncwarp();
        if (lane < G::KA)
          ptx::tma_load_2d(sm + G::V_OFF + sv * G::KTILE + lane * 16384, &tv, &v_full[sv], col0 + 64 * lane, slot);
      }
    }
  } else if (warp == 1) {
    {  // the converged warp runs the issue loop; one elected lane issues each MMA and commit
      constexpr uint32_t id_s = ptx::idesc_bf16_f32(128, DKT, false, false);
      constexpr uint32_t id_dq = ptx::idesc_bf16_f32(128, HD, false, true);
      bool ok = ptx::mbar_wait_warp(q_full, 0, err);
      // S_j = Q K_j^T and dP_j = dO V_j^T into the TMEM buffer, once both warpgroups read tile j-1's
      auto issue_s = [&](int j) {
        const int sk = j % NK, sv = j % NV;
        if (!ptx::mbar_wait_warp(&k_full[sk], (j / NK) & 1, err)) return false;
        if (!ptx::mbar_wait_warp(&v_full[sv], (j / NV) & 1, err)) return false;
        if (j >= 1 && !ptx::mbar_wait_warp(s_empty, (j - 1) & 1, err)) return false;
        ptx::tc_fence_after();
        const uint32_t k_addr = ptx::smem_u32(sm + G::K_OFF + sk * G::KTILE);
        const uint32_t v_addr = ptx::smem_u32(sm + G::V_OFF + sv * G::KTILE);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {  // K-steps of 16 along head_dim: atom ks / 4, offset ks % 4
          const uint32_t boff = (ks / 4) * 16384 + (ks % 4) * 32;
          ptx::umma_bf16_ts_elect(t_s, t_q + ks * 8, sdesc(k_addr + boff, 16, 1024, 2), id_s, ks > 0);
          ptx::umma_bf16_ts_elect(t_dp, t_do + ks * 8, sdesc(v_addr + boff, 16, 1024, 2), id_s, ks > 0);
        }
        ptx::umma_commit_elect(s_full);
        ptx::umma_commit_elect(&v_empty[sv]);  // V_j is not read again
        return true;
      };
      if (ok && ntiles > 0) ok = issue_s(0);
      for (int j = 0; ok && j < ntiles; ++j) {
        if (j + 1 < ntiles && !(ok = issue_s(j + 1))) break;
        if (!(ok = ptx::mbar_wait_warp(&ds_full[j & 1], (j / 2) & 1, err))) break;
        ptx::tc_fence_after();
        const int sk = j % NK;
        const uint32_t k_addr = ptx::smem_u32(sm + G::K_OFF + sk * G::KTILE);
        const uint32_t ds_addr = ptx::smem_u32(sm + G::DS_OFF + (j & 1) * G::DS_BYTES);
#pragma unroll
        for (int kk = 0; kk < DKT / 16; ++kk)  // dQ += dS_j K_j; K MN-major: atoms 16384 bytes apart (LBO)
          ptx::umma_bf16_elect(t_dq, sdesc(ds_addr + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024, 2),
                               sdesc(k_addr + kk * 2048, 16384, 1024, 2), id_dq, (j > 0 || kk > 0) ? 1u : 0u);
        ptx::umma_commit_elect(&k_empty[sk]);
        ptx::umma_commit_elect(&ds_free[j & 1]);
      }
      ptx::umma_commit_elect(dq_full);
      ptx::mbar_drain(dq_full, 0);
    }
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;  // this warpgroup owns key columns 64g .. 64g+63
    const int q = warp & 3;         // TMEM lane quarter
    const int r = q * 32 + lane;
    const int64_t p = q0 + r;
    const bool row_ok = p <= qlast;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const float L2E = 1.4426950408889634f;
    const float sl2 = a.scale * L2E;
    const int64_t i = p - a.p0;
    const float lse2 = row_ok ? a.lse[(int64_t)h * a.ld_lse + i] * L2E : 0.f;
    const float Di = row_ok ? a.D[(int64_t)h * a.ld_lse + i] : 0.f;
    {  // warpgroup 0 writes this row of Q, warpgroup 1 the row of dO, as packed bf16 pairs
      const bf16* src = g == 0 ? reinterpret_cast<const bf16*>(a.q) + i * a.ldq + col0
                               : reinterpret_cast<const bf16*>(a.dout) + i * a.lddo + col0;
      const uint32_t dst = (g == 0 ? t_q : t_do) + lane_off;
#pragma unroll
      for (int c = 0; c < HD / 2; c += 8) {  // 8 columns = 16 bf16 = two 16-byte loads
        uint4 u0 = make_uint4(0u, 0u, 0u, 0u), u1 = u0;
        if (row_ok) {
          u0 = *reinterpret_cast<const uint4*>(src + 2 * c);
          u1 = *reinterpret_cast<const uint4*>(src + 2 * c + 8);
        }
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        ptx::tmem_st8(dst + c, w);
      }
      tmem_st_wait();
      ptx::tc_fence_before();
      ptx::mbar_arrive(q_full);
    }
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int64_t j0 = j_begin + (int64_t)j * DKT + 64 * g;  // position of this warpgroup's first key
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(s_full, j & 1, err));
      if (!ok) break;
      ptx::tc_fence_after();
      float sv[64], dp[64];
      {
        uint32_t rs[64], rd[64];
        ptx::tmem_ld64(t_s + 64 * g + lane_off, rs);
        ptx::tmem_ld64(t_dp + 64 * g + lane_off, rd);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          sv[e] = __uint_as_float(rs[e]);
          dp[e] = __uint_as_float(rd[e]);
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(s_empty);
      if (j >= 2) {  // dS buffer j&1 is free once dQ_{j-2} consumed it
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&ds_free[j & 1], ((j - 2) / 2) & 1, err));
        if (!ok) break;
      }
      const int64_t lo = p - a.window + 1 - j0, hi = p - j0;
      if (!(row_ok && lo <= 0 && hi >= 63)) {  // edge tile: masked scores give P = 0
#pragma unroll
        for (int c = 0; c < 64; ++c) sv[c] = (row_ok && c >= lo && c <= hi) ? sv[c] : -INFINITY;
      }
      uint8_t* drow = sm + G::DS_OFF + (j & 1) * G::DS_BYTES + g * 16384 + r * 128;
#pragma unroll
      for (int gg = 0; gg < 8; ++gg) {  // granules of 8 keys
        float ds[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = gg * 8 + e;
          const float pr = ex2(fmaf(sv[c], sl2, -lse2));
          ds[e] = pr * (dp[c] - Di);
        }
        __nv_bfloat162 b0 = __floats2bfloat162_rn(ds[0], ds[1]), b1 = __floats2bfloat162_rn(ds[2], ds[3]);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(ds[4], ds[5]), b3 = __floats2bfloat162_rn(ds[6], ds[7]);
        *reinterpret_cast<uint4*>(drow + ((gg ^ (r & 7)) << 4)) =
            make_uint4(*reinterpret_cast<uint32_t*>(&b0), *reinterpret_cast<uint32_t*>(&b1),
                       *reinterpret_cast<uint32_t*>(&b2), *reinterpret_cast<uint32_t*>(&b3));
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&ds_full[j & 1]);
    }
    if (ok) ok = ptx::mbar_wait(dq_full, 0, err);
    if (__all_sync(0xffffffffu, ok)) {
      ptx::tc_fence_after();
      bf16* out = reinterpret_cast<bf16*>(a.dq) + i * a.lddq + col0;
      // warpgroup g writes the 16-column groups of parity g
#pragma unroll
      for (int c = 16 * g; c < HD; c += 32) {
        uint32_t o[16];
        tmem_ld16(t_dq + c + lane_off, o);
        ptx::tmem_ld_wait();
        if (row_ok) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            __nv_bfloat162 t2 = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * a.scale,
                                                      __uint_as_float(o[2 * e + 1]) * a.scale);
            pk[e] = *reinterpret_cast<uint32_t*>(&t2);
          }
          *reinterpret_cast<uint4*>(out + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(out + c + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// Backward, dk/dv part for the chunk's own keys (earlier keys are constants):
//   dV_j = sum_i P_ij dO_i,  dK_j = scale * sum_i dS_ij Q_i  over queries i >= j in the chunk.
// CTA = 128 keys x one head; query tiles of 128 from the key tile to the end of the chunk.
//   warp 0      TMA: K, V once; Q and dO tiles (2 stages)
//   warp 1      TMEM owner; lane 0 issues S^T = K Q^T and dP^T = V dO^T (128 + 128
//               columns), then dV += P^T dO and dK += dS^T Q (head_dim columns each)
//   warps 4..7  one key row per thread: P^T = exp(S^T*scale - lse_i), dS^T = P^T o
//               (dP^T - D_i), written as K-major (query-contiguous) swizzled operands
template <int HD>
struct KVGeo {
  static constexpr int A = HD / 64;
  static constexpr int R = HD % 64;
  static constexpr int RB = R * 2;
  static constexpr int TILE = 128 * HD * 2;    // any 128-row tile
  static constexpr int REM = A * 16384;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = TILE;
  static constexpr int QDST = HD <= 96 ? 2 : 1;  // Q/dO stages (shared memory bound at head_dim 128)
  static constexpr int QD_OFF = 2 * TILE;      // stage s: Q at QD_OFF + s*2*TILE, dO after it
  static constexpr int PT_OFF = QD_OFF + QDST * 2 * TILE;
  static constexpr int OP_BYTES = 128 * 128 * 2;  // P^T or dS^T tile (two 64-query atoms)
  static constexpr int DST_OFF = PT_OFF + OP_BYTES;
  static constexpr int LD_OFF = DST_OFF + OP_BYTES;  // lse*log2e [128] then D [128], fp32
  static constexpr int BAR_OFF = LD_OFF + 1024;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
};

template <int HD>
__global__ void __launch_bounds__(256, 1)
    swa_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tq_r,
                           const __grid_constant__ CUtensorMap tdo, const __grid_constant__ CUtensorMap tdo_r,
                           const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tk_r,
                           const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tv_r,
                           SwaArgs a, int* err) {
  using G = KVGeo<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + G::BAR_OFF);
  uint64_t* kv_full = bars + 0;
  uint64_t* qd_full = bars + 1;   // [2]
  uint64_t* qd_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* s_read = bars + 6;    // 128 arrivals: S^T/dP^T read and P^T/dS^T written
  uint64_t* pv_done = bars + 7;   // dV/dK products of the tile done (operands free)
  uint64_t* o_full = bars + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
  float* lse_s = reinterpret_cast<float*>(sm + G::LD_OFF);
  float* d_s = lse_s + 128;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t kb0 = (int64_t)blockIdx.x * 128;                   // first key row (chunk-local)
  const int64_t klast = imin64(kb0 + 128, a.n) - 1;
  const int64_t qend = imin64(a.n, klast + a.window);              // queries i < qend can see some key
  const int ntiles = (int)((qend - kb0 + 127) / 128);
  const int col0 = h * HD;

  if (threadIdx.x == 0) {
    ptx::mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&qd_full[s], 1);
      ptx::mbar_init(&qd_empty[s], 1);
    }
    ptx::mbar_init(s_full, 1);
    ptx::mbar_init(s_read, 128);
    ptx::mbar_init(pv_done, 1);
    ptx::mbar_init(o_full, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s = tmem, t_dp = tmem + 128, t_dv = tmem + 256, t_dk = tmem + 384;

  if (warp == 0) {
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(kv_full, 2 * G::TILE);
      const int slot = (int)((a.p0 + kb0) % a.ring);
      load_rows<HD>(sm + G::K_OFF, &tk, &tk_r, kv_full, col0, slot, 16384, G::REM);
      load_rows<HD>(sm + G::V_OFF, &tv, &tv_r, kv_full, col0, slot, 16384, G::REM);
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % G::QDST;
        if (!ptx::mbar_wait(&qd_empty[s], ((t / G::QDST) & 1) ^ 1, err)) break;
        ptx::mbar_arrive_expect_tx(&qd_full[s], 2 * G::TILE);
        const int qrow = (int)(kb0 + (int64_t)t * 128);
        uint8_t* qd = sm + G::QD_OFF + s * 2 * G::TILE;
        load_rows<HD>(qd, &tq, &tq_r, &qd_full[s], col0, qrow, 16384, G::REM);
        load_rows<HD>(qd + G::TILE, &tdo, &tdo_r, &qd_full[s], col0, qrow, 16384, G::REM);
      }
    }
  } else if (warp == 1) {
    {  // the converged warp runs the issue loop; one elected lane issues each MMA and commit
      constexpr uint32_t id_s = ptx::idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_o64 = ptx::idesc_bf16_f32(128, 64, false, true);
      constexpr uint32_t id_or = ptx::idesc_bf16_f32(128, G::R > 0 ? G::R : 16, false, true);
      constexpr uint32_t rl = rem_swizzle_layout(G::R);
      const uint32_t k_addr = ptx::smem_u32(sm + G::K_OFF), v_addr = ptx::smem_u32(sm + G::V_OFF);
      const uint32_t pt_addr = ptx::smem_u32(sm + G::PT_OFF), dst_addr = ptx::smem_u32(sm + G::DST_OFF);
      bool ok = ptx::mbar_wait_warp(kv_full, 0, err);
      for (int t = 0; ok && t < ntiles; ++t) {
        const int s = t % G::QDST;
        if (!(ok = ptx::mbar_wait_warp(&qd_full[s], (t / G::QDST) & 1, err))) break;
        ptx::tc_fence_after();
        const uint32_t q_addr = ptx::smem_u32(sm + G::QD_OFF + s * 2 * G::TILE), do_addr = q_addr + G::TILE;
        // S^T = K Q^T and dP^T = V dO^T (K over head_dim)
        int step = 0;
#pragma unroll
        for (int at = 0; at < G::A; ++at)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk, ++step) {
            ptx::umma_bf16_elect(t_s, sdesc(k_addr + at * 16384 + kk * 32, 16, 1024, 2),
                           sdesc(q_addr + at * 16384 + kk * 32, 16, 1024, 2), id_s, step > 0);
            ptx::umma_bf16_elect(t_dp, sdesc(v_addr + at * 16384 + kk * 32, 16, 1024, 2),
                           sdesc(do_addr + at * 16384 + kk * 32, 16, 1024, 2), id_s, step > 0);
          }
        if constexpr (G::R > 0) {
#pragma unroll
          for (int kk = 0; kk < G::R / 16; ++kk, ++step) {
            ptx::umma_bf16_elect(t_s, sdesc(k_addr + G::REM + kk * 32, 16, 8 * G::RB, rl),
                           sdesc(q_addr + G::REM + kk * 32, 16, 8 * G::RB, rl), id_s, step > 0);
            ptx::umma_bf16_elect(t_dp, sdesc(v_addr + G::REM + kk * 32, 16, 8 * G::RB, rl),
                           sdesc(do_addr + G::REM + kk * 32, 16, 8 * G::RB, rl), id_s, step > 0);
          }
        }
        ptx::umma_commit_elect(s_full);
        if (!(ok = ptx::mbar_wait_warp(s_read, t & 1, err))) break;
        ptx::tc_fence_after();
        // dV += P^T dO and dK += dS^T Q (K over the tile's 128 queries)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t pd = sdesc(pt_addr + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024, 2);
          const uint64_t dd = sdesc(dst_addr + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024, 2);
          const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
#pragma unroll
          for (int at = 0; at < G::A; ++at) {
            ptx::umma_bf16_elect(t_dv + 64 * at, pd, sdesc(do_addr + at * 16384 + kk * 2048, 16, 1024, 2), id_o64, acc);
            ptx::umma_bf16_elect(t_dk + 64 * at, dd, sdesc(q_addr + at * 16384 + kk * 2048, 16, 1024, 2), id_o64, acc);
          }
          if constexpr (G::R > 0) {
            ptx::umma_bf16_elect(t_dv + 64 * G::A, pd, sdesc(do_addr + G::REM + kk * 16 * G::RB, 16, 8 * G::RB, rl), id_or,
                           acc);
            ptx::umma_bf16_elect(t_dk + 64 * G::A, dd, sdesc(q_addr + G::REM + kk * 16 * G::RB, 16, 8 * G::RB, rl), id_or,
                           acc);
          }
        }
        ptx::umma_commit_elect(&qd_empty[s]);
        ptx::umma_commit_elect(pv_done);
      }
      ptx::umma_commit_elect(o_full);
      ptx::mbar_drain(o_full, 0);
    }
  } else if (warp >= 4) {
    const int r = (warp - 4) * 32 + lane;     // key row in the tile (== TMEM lane)
    const int64_t jl = kb0 + r;               // chunk-local key row
    const bool key_ok = jl < a.n;
    const uint32_t lane_off = (uint32_t)((warp - 4) * 32) << 16;
    const float L2E = 1.4426950408889634f;
    const float sl2 = a.scale * L2E;
    bool ok = true;
    for (int t = 0; t < ntiles; ++t) {
      const int64_t qb0 = kb0 + (int64_t)t * 128;
      ok = ptx::mbar_wait(s_full, t & 1, err);
      if (t > 0 && ok) ok = ptx::mbar_wait(pv_done, (t - 1) & 1, err);  // P^T/dS^T buffers free
      // all 128 key-row threads agree before the named barrier below (no one waits alone)
      ok = bar_and(1, 128, ok);
      if (!ok) break;
      // per-query statistics of this tile (thread r fetches query qb0 + r)
      {
        const int64_t i = qb0 + r;
        const bool q_ok = i < a.n;
        lse_s[r] = q_ok ? a.lse[(int64_t)h * a.ld_lse + i] * L2E : INFINITY;  // +inf: P = 0
        d_s[r] = q_ok ? a.D[(int64_t)h * a.ld_lse + i] : 0.f;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      ptx::tc_fence_after();
      uint8_t* prow = sm + G::PT_OFF + r * 128;
      uint8_t* drow = sm + G::DST_OFF + r * 128;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        float sv[64], dp[64];
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          uint32_t rs[32], rd[32];
          ptx::tmem_ld32(t_s + half * 64 + c + lane_off, rs);
          ptx::tmem_ld32(t_dp + half * 64 + c + lane_off, rd);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            sv[c + e] = __uint_as_float(rs[e]);
            dp[c + e] = __uint_as_float(rd[e]);
          }
        }
        // query i = qb0 + half*64 + c sees key jl iff jl <= i < jl + window
        const int64_t lo = jl - qb0 - half * 64, hi = jl + a.window - 1 - qb0 - half * 64;
        if (!(key_ok && lo <= 0 && hi >= 63)) {
#pragma unroll
          for (int c = 0; c < 64; ++c) sv[c] = (key_ok && c >= lo && c <= hi) ? sv[c] : -INFINITY;
        }
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          float pv[8], dv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = g * 8 + e, q = half * 64 + c;
            pv[e] = ex2(fmaf(sv[c], sl2, -lse_s[q]));
            dv[e] = pv[e] * (dp[c] - d_s[q]);
          }
          uint4 w, x;
          __nv_bfloat162 p0 = __floats2bfloat162_rn(pv[0], pv[1]), p1 = __floats2bfloat162_rn(pv[2], pv[3]);
          __nv_bfloat162 p2 = __floats2bfloat162_rn(pv[4], pv[5]), p3 = __floats2bfloat162_rn(pv[6], pv[7]);
          __nv_bfloat162 d0 = __floats2bfloat162_rn(dv[0], dv[1]), d1 = __floats2bfloat162_rn(dv[2], dv[3]);
          __nv_bfloat162 d2 = __floats2bfloat162_rn(dv[4], dv[5]), d3 = __floats2bfloat162_rn(dv[6], dv[7]);
          w.x = *reinterpret_cast<uint32_t*>(&p0);
          w.y = *reinterpret_cast<uint32_t*>(&p1);
          w.z = *reinterpret_cast<uint32_t*>(&p2);
          w.w = *reinterpret_cast<uint32_t*>(&p3);
          x.x = *reinterpret_cast<uint32_t*>(&d0);
          x.y = *reinterpret_cast<uint32_t*>(&d1);
          x.z = *reinterpret_cast<uint32_t*>(&d2);
          x.w = *reinterpret_cast<uint32_t*>(&d3);
          const int off = half * 16384 + ((g ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(prow + off) = w;
          *reinterpret_cast<uint4*>(drow + off) = x;
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(s_read);
    }
    if (ok) ok = ptx::mbar_wait(o_full, 0, err);
    if (__all_sync(0xffffffffu, ok)) {
      ptx::tc_fence_after();
      bf16* ov = reinterpret_cast<bf16*>(a.dv) + jl * a.lddkv + col0;
      bf16* ok_ = reinterpret_cast<bf16*>(a.dk) + jl * a.lddkv + col0;
#pragma unroll
      for (int c = 0; c < HD; c += 16) {
        uint32_t v[16], kx[16];
        tmem_ld16(t_dv + c + lane_off, v);
        tmem_ld16(t_dk + c + lane_off, kx);
        ptx::tmem_ld_wait();
        if (key_ok) {
          uint32_t pv_[8], pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            __nv_bfloat162 tv2 = __floats2bfloat162_rn(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
            __nv_bfloat162 tk2 = __floats2bfloat162_rn(__uint_as_float(kx[2 * e]) * a.scale,
                                                       __uint_as_float(kx[2 * e + 1]) * a.scale);
            pv_[e] = *reinterpret_cast<uint32_t*>(&tv2);
            pk[e] = *reinterpret_cast<uint32_t*>(&tk2);
          }
          *reinterpret_cast<uint4*>(ov + c) = make_uint4(pv_[0], pv_[1], pv_[2], pv_[3]);
          *reinterpret_cast<uint4*>(ov + c + 8) = make_uint4(pv_[4], pv_[5], pv_[6], pv_[7]);
          *reinterpret_cast<uint4*>(ok_ + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(ok_ + c + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode() {
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

// bf16 [rows, cols] with row pitch ld; box = box_cols x 128 rows; swizzle by box width.
int tmap(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int64_t ld, int box_cols, int box_rows = 128) {
  EncodeTiledFn enc = encode();
  if (!enc) return set_error(TTT_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || ((ld * 2) & 15))
    return set_error(TTT_ERR_INVALID_ARG, "attention: operands must be 16-byte aligned");
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1u, 1u};
  const CUtensorMapSwizzle sw = box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                 : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(TTT_ERR_CUDA, "attention tensor map: " + std::to_string((int)r));
  return TTT_OK;
}

template <int HD>
int launch(const SwaTcPlan& p, const SwaArgs& a, cudaStream_t s, int* err) {
  using G = Geo<HD>;
  auto fn = &swa_fwd_tc_kernel<HD>;
  {
    static std::mutex mu;
    static std::set<int> done;
    int dev = 0;
    TTT_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lock(mu);
    if (!done.count(dev)) {
      TTT_CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM));
      done.insert(dev);
    }
  }
  dim3 grid(ceil_div(a.n, QT), a.heads);
  fn<<<grid, 384, G::SMEM, s>>>(p.q128, p.qr, p.k128, p.kr, p.v128, a, err);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}


template <int HD>
int launch_bwd_dq(const SwaTcBwdPlan& p, const SwaArgs& a, cudaStream_t s, int* err) {
  using G = DGeo<HD>;
  auto fn = &swa_bwd_dq128_kernel<HD>;
  {
    static std::mutex mu;
    static std::set<int> done;
    int dev = 0;
    TTT_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lock(mu);
    if (!done.count(dev)) {
      TTT_CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM));
      done.insert(dev);
    }
  }
  dim3 grid(ceil_div(a.n, QT), a.heads);
  fn<<<grid, 384, G::SMEM, s>>>(p.k128, p.v128, a, err);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <int HD>
int launch_bwd_dkdv(const SwaTcBwdPlan& p, const SwaArgs& a, cudaStream_t s, int* err) {
  using G = KVGeo<HD>;
  auto fn = &swa_bwd_dkdv_tc_kernel<HD>;
  {
    static std::mutex mu;
    static std::set<int> done;
    int dev = 0;
    TTT_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lock(mu);
    if (!done.count(dev)) {
      TTT_CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM));
      done.insert(dev);
    }
  }
  dim3 grid(ceil_div(a.n, 128), a.heads);
  fn<<<grid, 256, G::SMEM, s>>>(p.q128, p.qr, p.do128, p.dor, p.k128, p.kr128, p.v128, p.vr128, a, err);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

}  // namespace

int swa_tc_bwd_prepare(SwaTcBwdPlan* p, int heads, int head_dim, const void* q, const void* dout, int64_t rows,
                       int64_t ld, const void* k, const void* v, int64_t ring, int64_t ldkv) {
  if (!swa_tc_supported(head_dim)) return set_error(TTT_ERR_UNSUPPORTED, "attention: head_dim not supported");
  if (ring % 128) return set_error(TTT_ERR_INVALID_ARG, "attention: ring slots must be a multiple of 128");
  p->head_dim = head_dim;
  p->ring = ring;
  const int64_t cols = (int64_t)heads * head_dim;
  const int rem = head_dim % 64;
  int rc = tmap(&p->q128, q, rows, cols, ld, 64);
  if (!rc) rc = tmap(&p->do128, dout, rows, cols, ld, 64);
  if (!rc) rc = tmap(&p->k64, k, ring, cols, ldkv, 64, 64);
  if (!rc) rc = tmap(&p->v64, v, ring, cols, ldkv, 64, 64);
  if (!rc) rc = tmap(&p->k128, k, ring, cols, ldkv, 64, 128);
  if (!rc) rc = tmap(&p->v128, v, ring, cols, ldkv, 64, 128);
  if (rc) return rc;
  if (rem) {
    rc = tmap(&p->qr, q, rows, cols, ld, rem);
    if (!rc) rc = tmap(&p->dor, dout, rows, cols, ld, rem);
    if (!rc) rc = tmap(&p->kr, k, ring, cols, ldkv, rem, 64);
    if (!rc) rc = tmap(&p->vr, v, ring, cols, ldkv, rem, 64);
    if (!rc) rc = tmap(&p->kr128, k, ring, cols, ldkv, rem, 128);
    if (!rc) rc = tmap(&p->vr128, v, ring, cols, ldkv, rem, 128);
  } else {
    p->qr = p->q128;
    p->dor = p->do128;
    p->kr = p->k64;
    p->vr = p->v64;
    p->kr128 = p->k128;
    p->vr128 = p->v128;
  }
  return rc;
}

bool swa_tc_dkdv_supported(const SwaArgs& a) { return a.p0 % 128 == 0 && a.ring % 128 == 0; }

int swa_tc_backward_dkdv(const SwaTcBwdPlan& p, const SwaArgs& a, cudaStream_t s, int* err) {
  if (a.ring != p.ring || a.head_dim != p.head_dim) return set_error(TTT_ERR_INVALID_ARG, "attention: plan mismatch");
  if (!swa_tc_dkdv_supported(a)) return set_error(TTT_ERR_INVALID_ARG, "attention: dk/dv needs 128-aligned chunks");
  switch (a.head_dim) {
    case 64: return launch_bwd_dkdv<64>(p, a, s, err);
    case 80: return launch_bwd_dkdv<80>(p, a, s, err);
    case 96: return launch_bwd_dkdv<96>(p, a, s, err);
    case 128: return launch_bwd_dkdv<128>(p, a, s, err);
  }
  return set_error(TTT_ERR_UNSUPPORTED, "attention (tensor cores): head_dim must be 64, 80, 96 or 128");
}

int swa_tc_backward_dq(const SwaTcBwdPlan& p, const SwaArgs& a, cudaStream_t s, int* err) {
  if (a.ring != p.ring || a.head_dim != p.head_dim) return set_error(TTT_ERR_INVALID_ARG, "attention: plan mismatch");
  switch (a.head_dim) {
    case 64: return launch_bwd_dq<64>(p, a, s, err);
    case 80: return launch_bwd_dq<80>(p, a, s, err);
    case 96: return launch_bwd_dq<96>(p, a, s, err);
    case 128: return launch_bwd_dq<128>(p, a, s, err);
  }
  return set_error(TTT_ERR_UNSUPPORTED, "attention (tensor cores): head_dim must be 64, 80, 96 or 128");
}

namespace {
}  // namespace

bool swa_tc_supported(int head_dim) {
  return head_dim == 64 || head_dim == 80 || head_dim == 96 || head_dim == 128;
}

int swa_tc_prepare(SwaTcPlan* p, int heads, int head_dim, const void* q, int64_t q_rows, int64_t ldq, const void* k,
                   const void* v, int64_t ring, int64_t ldkv) {
  if (!swa_tc_supported(head_dim)) return set_error(TTT_ERR_UNSUPPORTED, "attention: head_dim not supported");
  if (ring % KT) return set_error(TTT_ERR_INVALID_ARG, "attention: ring slots must be a multiple of 128");
  p->head_dim = head_dim;
  p->ring = ring;
  const int64_t cols = (int64_t)heads * head_dim;
  const int rem = head_dim % 64;
  int rc = tmap(&p->q128, q, q_rows, cols, ldq, 64);
  if (!rc) rc = tmap(&p->k128, k, ring, cols, ldkv, 64);
  if (!rc) rc = tmap(&p->k64, k, ring, cols, ldkv, 64, 64);
  if (!rc) rc = tmap(&p->v128, v, ring, cols, ldkv, 64);
  if (rc) return rc;
  if (rem) {
    rc = tmap(&p->qr, q, q_rows, cols, ldq, rem);
    if (!rc) rc = tmap(&p->kr, k, ring, cols, ldkv, rem);
    if (!rc) rc = tmap(&p->kr64, k, ring, cols, ldkv, rem, 64);
  } else {
    p->qr = p->q128;
    p->kr = p->k128;
    p->kr64 = p->k64;
  }
  return rc;
}

namespace {
constexpr int kExpPolyDefault = 2;  // of every 8 groups of 8 keys (fixed-shift path)

template <int HD, int EMU>
int launch_fx(const SwaTcPlan& p, const SwaArgs& a, cudaStream_t s, int* err) {
  using G = FxGeo<HD>;
  auto fn = &swa_fwd_fx_kernel<HD, EMU, 2>;
  {
    static std::mutex mu;
    static std::set<int> done;
    int dev = 0;
    TTT_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lock(mu);
    if (!done.count(dev)) {
      TTT_CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM));
      done.insert(dev);
    }
  }
  dim3 grid(ceil_div(a.n, QT), a.heads);
  fn<<<grid, 384, G::SMEM, s>>>(p.k128, p.kr, p.v128, a, err);
  TTT_CUDA_TRY(cudaGetLastError());
  return TTT_OK;
}

template <int HD>
int launch_emu(const SwaTcPlan& p, const SwaArgs& a, int fixed, cudaStream_t s, int* err) {
  if (!fixed) return launch<HD>(p, a, s, err);
  switch (a.exp_poly < 0 ? kExpPolyDefault : a.exp_poly) {
    case 0: return launch_fx<HD, 0>(p, a, s, err);
    case 2: return launch_fx<HD, 2>(p, a, s, err);
    case 4: return launch_fx<HD, 4>(p, a, s, err);
  }
  return set_error(TTT_ERR_INVALID_ARG, "attention: polynomial share must be 0, 2 or 4 of 8");
}
}  // namespace

bool swa_fixed_shift_ok(const SwaArgs& a) {
  const double m = (double)a.scale * 1.4426950408889634 * a.q_norm_max * a.k_norm_max * 1.01;
  return a.q_norm_max > 0.f && a.k_norm_max > 0.f && m <= 48.0;
}

int swa_tc_forward(const SwaTcPlan& p, const SwaArgs& a, cudaStream_t s, int* err) {
  if (a.ring != p.ring || a.head_dim != p.head_dim) return set_error(TTT_ERR_INVALID_ARG, "attention: plan mismatch");
  const int fx = swa_fixed_shift_ok(a) ? 1 : 0;
  switch (a.head_dim) {
    case 64: return launch_emu<64>(p, a, fx, s, err);
    case 80: return launch_emu<80>(p, a, fx, s, err);
    case 96: return launch_emu<96>(p, a, fx, s, err);
    case 128: return launch_emu<128>(p, a, fx, s, err);
  }
  return set_error(TTT_ERR_UNSUPPORTED, "attention (tensor cores): head_dim must be 64, 80, 96 or 128");
}

}  // namespace ttt
