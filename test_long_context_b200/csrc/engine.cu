// The TTT-E2E prefill engine behind include/ttt.h.
//
// Schedule of ttt_prefill (算法 1 of the reading notes, eq. (9)):
//   Blocks 0 .. L-n_u-1 have no fast weights, so their outputs depend only
//   on the tokens.  They run over a super-chunk of S = spc*b positions at a
//   time (large-M GEMMs), with their own KV rings of S + k slots.
//   Blocks L-n_u .. L-1 then run chunk by chunk (b positions): forward with
//   the current fast weights, per-token losses recorded, then - for every
//   full chunk - the backward through these blocks and one SGD step on each
//   block's fast MLP, applied right after that block's data gradients.
// Everything in the loop is device work on one stream; the host only
// enqueues.
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <memory>
#include <string>
#include <vector>

#include "../../include/ttt.h"
#include "attention.cuh"
#include "attention_tc.cuh"
#include "decode.cuh"
#include "elementwise.cuh"
#include "gemm.cuh"

struct ttt_ctx {
  virtual ~ttt_ctx() = default;
  virtual int prefill(const int32_t* tok, int64_t T, float* losses, float* const* fast_out) = 0;
  virtual int decode(int64_t count, int32_t* tokens, float* losses) = 0;
  virtual int reset() = 0;
  virtual int sync() = 0;
  virtual int timing_enable(bool on) = 0;
  virtual int timing_read(int kc, double* ms, int64_t* n, double* flops) = 0;
  std::string last_error = "no error";
  int64_t launches = 0;
};

namespace ttt {
namespace {

// Device allocations owned by a context, released together.
struct Arena {
  std::vector<void*> blocks;
  cudaStream_t stream = nullptr;
  ~Arena() {
    for (void* p : blocks) cudaFree(p);
  }
  template <typename T>
  int alloc(T** out, int64_t count) {
    void* p = nullptr;
    const size_t bytes = (size_t)(count > 0 ? count : 1) * sizeof(T);
    cudaError_t e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return set_error(TTT_ERR_OOM, "cudaMalloc of " + std::to_string(bytes) + " bytes failed");
    }
    blocks.push_back(p);
    e = cudaMemsetAsync(p, 0, bytes, stream);
    if (e != cudaSuccess) return set_cuda_error(e, "cudaMemsetAsync", __FILE__, __LINE__);
    *out = reinterpret_cast<T*>(p);
    return TTT_OK;
  }
};

#define TRY(expr)                 \
  do {                            \
    int rc_ = (expr);             \
    if (rc_ != TTT_OK) return rc_; \
  } while (0)

template <typename T>
struct ActTraits;
template <>
struct ActTraits<float> {
  static constexpr bool bf = false;
  static constexpr int store_epi = EPI_STORE_F32;
};
template <>
struct ActTraits<bf16> {
  static constexpr bool bf = true;
  static constexpr int store_epi = EPI_STORE_BF16;
};

// One GEMM of the schedule, with its tensor maps built once (bf16 mode).
struct Gemm {
  GemmShape shape;
  int epi = 0;
  EpiArgs args;
  TcGemm tc;
  bool bf = false;
  int64_t split = 1;  // deterministic split-K count (bf16 mode)
  const char* label = "gemm";
  // the product recomputes values the forward already had (the LM-head
  // logits of the backward): its flops are not algorithmic work
  bool recompute = false;
};

// Event timing of launches, per kernel class (opt-in).  Back-to-back launches
// share one event per boundary: a launch's start is the previous launch's end
// event while nothing else was enqueued in between (`chain`), so a launch costs
// one event record instead of two and the per-launch times add up to the
// stream's elapsed time.
struct LaunchTimer {
  struct Rec {
    int kc;
    cudaEvent_t a, b;
    double flops;
    std::string label;
    bool own_a;  // `a` was recorded for this launch (else it is the previous launch's `b`)
  };
  struct Stat {
    double ms = 0, flops = 0;
    int64_t n = 0;
  };
  std::map<std::string, Stat> by_label;  // filled when `labels` is set (TTT_PROFILE=1)
  bool labels = false;
  bool on = false;
  std::vector<Rec> pending;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t chain = nullptr;  // end event of the last timed launch, if it is the stream's last operation
  double ms[TTT_KC_COUNT] = {}, flops[TTT_KC_COUNT] = {};
  int64_t n[TTT_KC_COUNT] = {};
  ~LaunchTimer() {
    for (auto& r : pending) {
      if (r.own_a) cudaEventDestroy(r.a);
      cudaEventDestroy(r.b);
    }
    for (auto e : pool) cudaEventDestroy(e);
  }
  // Something other than a timed launch is about to be enqueued: the next
  // timed launch records its own start event.
  void cut() { chain = nullptr; }
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  int drain() {
    for (auto& r : pending) {
      float t = 0.f;
      TTT_CUDA_TRY(cudaEventElapsedTime(&t, r.a, r.b));
      ms[r.kc] += t;
      flops[r.kc] += r.flops;
      n[r.kc] += 1;
      if (labels && !r.label.empty()) {
        Stat& st = by_label[r.label];
        st.ms += t;
        st.flops += r.flops;
        st.n += 1;
      }
      if (r.own_a) pool.push_back(r.a);
      pool.push_back(r.b);
    }
    pending.clear();
    chain = nullptr;  // its event is back in the pool
    return TTT_OK;
  }
  void clear() {
    for (int i = 0; i < TTT_KC_COUNT; ++i) ms[i] = flops[i] = 0, n[i] = 0;
    by_label.clear();
  }
  // TTT_PROFILE=1: per-label table on stderr (launches, ms, TFLOP/s) of what was timed.
  void report() const {
    if (!labels || by_label.empty()) return;
    fprintf(stderr, "[ttt profile] %-22s %8s %10s %9s\n", "label", "launches", "ms", "TFLOP/s");
    for (const auto& kv : by_label)
      fprintf(stderr, "[ttt profile] %-22s %8lld %10.3f %9.1f\n", kv.first.c_str(), (long long)kv.second.n,
              kv.second.ms, kv.second.ms > 0 ? kv.second.flops / kv.second.ms / 1e9 : 0.0);
  }
};

template <typename T>
class Engine final : public ttt_ctx {
 public:
  Engine(const ttt_config& cfg, const ttt_weights& w, float eta, int k, int b, int nu, cudaStream_t s)
      : cfg_(cfg), eta_(eta), k_(k), b_(b), nu_(nu), st_(s) {
    wt_ = w;
    layers_.assign(w.layers, w.layers + cfg.n_layers);
    fast_init_.assign(w.fast, w.fast + nu);
    wt_.layers = layers_.data();
    wt_.fast = fast_init_.data();
  }

  int init();
  int prefill(const int32_t* tok, int64_t T_, float* losses, float* const* fast_out) override;
  int decode(int64_t count, int32_t* tokens, float* losses) override;
  int reset() override;
  int sync() override;
  ~Engine() override {
    if (timer_.labels && cudaStreamSynchronize(st_) == cudaSuccess && timer_.drain() == TTT_OK) timer_.report();
  }
  int timing_enable(bool on) override {
    TTT_CUDA_TRY(cudaStreamSynchronize(st_));
    TRY(timer_.drain());
    timer_.report();  // TTT_PROFILE: what was timed since the last enable
    timer_.clear();
    timer_.on = on;
    return TTT_OK;
  }
  int timing_read(int kc, double* ms, int64_t* n, double* flops) override {
    if (kc < 0 || kc >= TTT_KC_COUNT) return set_error(TTT_ERR_INVALID_ARG, "ttt_timing_read: bad class");
    TTT_CUDA_TRY(cudaStreamSynchronize(st_));
    TRY(timer_.drain());
    if (ms) *ms = timer_.ms[kc];
    if (n) *n = timer_.n[kc];
    if (flops) *flops = timer_.flops[kc];
    return TTT_OK;
  }

 private:
  static constexpr bool BF = ActTraits<T>::bf;
  static constexpr int STORE = ActTraits<T>::store_epi;

  int prep(Gemm& g, int a_mn, MatView a, int b_mn, MatView b, int epi, const EpiArgs& args);
  // bf16 mode: add the second product A2 B2^T on output columns >= n_ext (re-plans split-K)
  int prep_ext(Gemm& g, MatView a2, MatView b2, int64_t n_ext);
  int run(Gemm& g, int64_t rows);  // rows overrides the M extent (chunk/super-chunk length)
  int bottom_layers(const int32_t* tok, int64_t s0, int64_t S);
  int chunk(const int32_t* tok, int64_t T_, int64_t p0, int64_t n, const float* x0, float* losses);
  // backward through the updated blocks and the SGD steps of the chunk at p0
  // (n rows of the per-chunk buffers, targets in tgt_, CE scale in scl_)
  // logits_stored: the forward kept this chunk's LM-head logits in logits_
  // (the prefill in bf16 mode); else they are recomputed per vocab chunk
  int chunk_backward(int64_t p0, int64_t n, bool logits_stored);
  // generation: the forward of position p (token in dtok_) through every
  // block, the greedy pick of the next token, and the chunk's update when p
  // is its last position
  int decode_position(int64_t p);
  // greedy pick from the final-norm output row hf (the LM head as a
  // matrix-vector product): next token -> dtok_, loss -> dloss_
  // hf: a final-norm output row; or (hf NULL) xres: the residual row, normalised
  // in the product's prologue and stored to h_out, its factor to r_out
  int head_pick(const T* hf, const float* xres, T* h_out, float* r_out, int32_t* tgt_row, float* lse_row);
  template <typename G>
  int gemv_run(const GemvArgs<T>& a, int epi, G&& bytes_of);
  // Launch `f` (returns a status); bracket it with events when timing is on.
  template <typename F>
  int timed(int kc, double flops, F&& f, const char* label = nullptr) {
    ++launches;
    if (trace_) return traced(kc, f);
    if (!timer_.on) return f();
    static const char* names[TTT_KC_COUNT] = {"gemm", "attn_fwd", "attn_bwd", "other", "norm", "rope", "decode"};
    cudaEvent_t a = timer_.chain;
    const bool own_a = a == nullptr;
    if (own_a) {
      a = timer_.get();
      TTT_CUDA_TRY(cudaEventRecord(a, st_));
    }
    const int rc = f();
    cudaEvent_t b = timer_.get();
    TTT_CUDA_TRY(cudaEventRecord(b, st_));
    timer_.chain = b;
    std::string lab;
    if (timer_.labels) lab = label ? std::string(label) : std::string(phase_) + "." + names[kc];
    timer_.pending.push_back({kc, a, b, flops, std::move(lab), own_a});
    return rc;
  }
  // TTT_TRACE=1: synchronise after every launch and log it to stderr (debugging aid).
  template <typename F>
  int traced(int kc, F&& f) {
    static const char* names[TTT_KC_COUNT] = {"gemm", "attn_fwd", "attn_bwd", "other", "norm", "rope", "decode"};
    if (trace_verbose_) fprintf(stderr, "[ttt trace] launching %lld %s\n", (long long)launches, names[kc]);
    cudaEvent_t a = timer_.get(), b = timer_.get();
    TTT_CUDA_TRY(cudaEventRecord(a, st_));
    const int rc = f();
    TTT_CUDA_TRY(cudaEventRecord(b, st_));
    const cudaError_t e = cudaStreamSynchronize(st_);
    float ms = 0.f;
    cudaEventElapsedTime(&ms, a, b);
    timer_.pool.push_back(a);
    timer_.pool.push_back(b);
    int h = 0;
    cudaMemcpy(&h, err_, sizeof(int), cudaMemcpyDeviceToHost);
    if (ms > trace_ms_ || h || e != cudaSuccess || rc != TTT_OK)
      fprintf(stderr, "[ttt trace] launch %lld %s %.3f ms rc=%d cuda=%d err_word=%d\n", (long long)launches,
              names[kc], ms, rc, (int)e, h);
    if (e != cudaSuccess) return set_cuda_error(e, "trace sync", __FILE__, __LINE__);
    return rc;
  }
  // Query-key pairs admitted by the window for queries p0 .. p0+n-1 (eq. (1)).
  double band_pairs(int64_t p0, int64_t n) const {
    const int64_t k = k_;
    double s = 0;
    // queries with p + 1 <= k see p + 1 keys, the rest see k
    const int64_t full_from = std::max<int64_t>(p0, k - 1);
    const int64_t e = p0 + n;
    if (full_from > p0) {
      const int64_t a = p0 + 1, z = std::min<int64_t>(full_from, e);  // keys p+1 for p in [p0, z)
      s += (double)(a + z) * (double)(z - p0) / 2.0;
    }
    if (e > full_from) s += (double)(e - full_from) * (double)k;
    return s;
  }
  SwaArgs swa_args(const T* q, int64_t n, int64_t p0, const T* kr, const T* vr, int64_t ring, T* o, float* lse,
                   int64_t ld_lse, int64_t layer) const {
    SwaArgs a;
    a.q_norm_max = qn_max_[layer];  // bounds from the block's QK-norm gains
    a.k_norm_max = kn_max_[layer];
    a.heads = (int)H_;
    a.head_dim = (int)HD_;
    a.n = n;
    a.p0 = p0;
    a.window = k_;
    a.scale = scale_;
    a.q = q;
    a.ldq = d_;
    a.k = kr;
    a.v = vr;
    a.ldkv = d_;
    a.ring = ring;
    a.o = o;
    a.ldo = d_;
    a.lse = lse;
    a.ld_lse = ld_lse;
    return a;
  }
  float* master_gu(int i) { return BF ? m_gu_[i] : reinterpret_cast<float*>(wgu_[nbot_ + i]) + 2 * f_ * d_; }
  float* master_d(int i) { return BF ? m_d_[i] : reinterpret_cast<float*>(wd_[nbot_ + i]) + f_; }
  int64_t master_d_ld() const { return BF ? f_ : 2 * f_; }

  ttt_config cfg_;
  float eta_;
  int k_, b_, nu_;
  cudaStream_t st_;
  ttt_weights wt_;
  std::vector<ttt_layer_weights> layers_;
  std::vector<ttt_fast_weights> fast_init_;
  Arena arena_;
  LaunchTimer timer_;
  bool trace_ = false, trace_verbose_ = false;
  const char* phase_ = "misc";  // label prefix of untagged launches under TTT_PROFILE
  float trace_ms_ = 0.f;
  bool fresh_ = true;
  int* err_ = nullptr;
  // generation state: the next position to process, whether dtok_ already
  // holds its token, and the chunk start of the last processed position
  bool prefilled_ = false, dec_ready_ = false;
  int64_t dec_pos_ = 0;
  int32_t* dtok_ = nullptr;
  float* dloss_ = nullptr;
  float* xd_ = nullptr;        // residual of the generated position through the blocks without fast weights
  float* adws_ = nullptr;      // single-query attention work space
  float* gvpart_ = nullptr;    // LM-head greedy-pick partials
  int64_t gvparts_ = 0;

  int64_t d_ = 0, f_ = 0, H_ = 0, HD_ = 0, V_ = 0, L_ = 0, nbot_ = 0;
  int64_t S_ = 0, R1_ = 0, R_ = 0, Vc_ = 0, nvc_ = 0, ce_tiles_ = 0;
  float scale_ = 1.f;

  // weights rearranged for the GEMMs
  std::vector<T*> wqkv_;   // [3d, d] per block
  std::vector<T*> wgu_;    // bottom: [2f, d]; top: [4f, d] (static | fast), interleaved gate/up
  std::vector<T*> wd_;     // top: [d, 2f] (static | fast); bottom: caller's [d, f]
  std::vector<float*> m_gu_, m_d_;        // fp32 masters (bf16 mode) per top block
  // bf16 mode: the fast shadow is a two-term bf16 pair hi + lo of the master
  // (hi inside wgu_/wd_, lo here), so the forward sees updates far below one
  // bf16 ulp of W
  std::vector<bf16*> gu_lo_, d_lo_;       // [2f, d] interleaved, [d, f]
  std::vector<float*> init_gu_, init_d_;  // W_init copies per top block
  // phase-1 buffers
  float* xs_ = nullptr;
  float2* rope_tab_ = nullptr;  // RoPE (cos, sin) of the current super-chunk's positions, from tab_p0_
  int64_t tab_p0_ = 0;
  T *hs_ = nullptr, *qkvs_ = nullptr, *qs_ = nullptr, *os_ = nullptr, *as_ = nullptr;
  float *rs_ = nullptr, *rqs_ = nullptr, *rks_ = nullptr, *lses_ = nullptr;
  std::vector<T*> kb_, vb_;  // bottom rings [R1, d]
  // top blocks, per block i
  std::vector<float*> xin_, r1_, xmid_, r2_, rq_, rk_, lse_;
  std::vector<T*> h_, qkv_, q_, o_, h2_, gu_, a_, kt_, vt_;
  float *xf_ = nullptr, *rf_ = nullptr;
  T* hf_ = nullptr;
  float *pmax_ = nullptr, *psum_ = nullptr, *zt_ = nullptr, *lsef_ = nullptr, *scl_ = nullptr;
  float* logits_ = nullptr;  // bf16 mode: the chunk's LM-head logits [b, V] (fp32), kept for the backward
  int32_t* tgt_ = nullptr;
  // backward
  float *dx_ = nullptr, *dxm_ = nullptr, *dhf_ = nullptr, *dh2_ = nullptr, *dh_ = nullptr, *Dbuf_ = nullptr;
  T *dx16_ = nullptr, *dxm16_ = nullptr, *dz_ = nullptr, *da_ = nullptr, *dgu_ = nullptr, *do_ = nullptr,
    *dqkv_ = nullptr;
  // GEMM plans
  std::vector<Gemm> g_bot_;  // 4 per bottom block: qkv, o, gu, down
  std::vector<Gemm> g_top_;  // 10 per top block: qkv, o, gu, down, da, dh2, wd, wgu, do, dh
  Gemm g_head_;
  std::vector<Gemm> g_ce_dz_, g_ce_dh_;
  // split-K workspace shared by every split GEMM (they run one after another on the stream)
  int64_t ws_floats_ = 0;
  float* ws_ = nullptr;
  int finalize_splits() {
    if (!ws_floats_) return TTT_OK;
    TRY(arena_.alloc(&ws_, ws_floats_));
    auto fix = [&](Gemm& g) { return g.split > 1 ? tc_gemm_set_split(&g.tc, g.split, ws_) : TTT_OK; };
    for (auto& g : g_bot_) TRY(fix(g));
    for (auto& g : g_top_) TRY(fix(g));
    TRY(fix(g_head_));
    for (auto& g : g_ce_dz_) TRY(fix(g));
    for (auto& g : g_ce_dh_) TRY(fix(g));
    return TTT_OK;
  }
  // tensor-core attention plans (bf16, supported head_dim)
  bool tc_attn_ = false;
  // per block: max|g| sqrt(head_dim) of the QK-norm gains, bounds on the norms
  // of the normalised query and key rows (read once, at init)
  std::vector<float> qn_max_, kn_max_;
  std::vector<SwaTcPlan> att_bot_, att_top_;
  std::vector<SwaTcBwdPlan> att_bwd_;
  int attn_fwd(const SwaTcPlan* plan, const SwaArgs& a) {
    if (tc_attn_) return swa_tc_forward(*plan, a, st_, err_);
    return swa_forward(a, BF, st_);
  }
};

template <typename T>
int Engine<T>::prep(Gemm& g, int a_mn, MatView a, int b_mn, MatView b, int epi, const EpiArgs& args) {
  g.shape.a_mn = a_mn;
  g.shape.b_mn = b_mn;
  g.shape.a = a;
  g.shape.b = b;
  g.epi = epi;
  g.args = args;
  g.bf = BF;
  if (BF) {
    g.tc.act_bf16 = 1;
    int bn = 0;
    const int64_t S = tc_split_plan(g.shape.M(), g.shape.N(), g.shape.K(), epi, &bn);
    TRY(tc_gemm_prepare(&g.tc, g.shape, epi, args, bn));
    if (S > 1) {
      g.split = S;
      ws_floats_ = std::max<int64_t>(ws_floats_, S * g.shape.M() * g.shape.N());
    }
  }
  return TTT_OK;
}

template <typename T>
int Engine<T>::prep_ext(Gemm& g, MatView a2, MatView b2, int64_t n_ext) {
  if (!BF) return TTT_OK;
  const int64_t K2 = g.shape.a_mn ? a2.rows : a2.cols;
  const int64_t M = g.shape.M(), N = g.shape.N(), K = g.shape.K();
  int bn = 0;
  int64_t S = n_ext == 0 ? tc_split_plan(M, N, K + K2, g.epi, &bn) : 1;
  if (n_ext > 0 && n_ext % tc_pick_bn(M, N, 0)) bn = 128;  // tiles must not straddle n_ext
  TRY(tc_gemm_prepare(&g.tc, g.shape, g.epi, g.args, bn));
  TRY(tc_gemm_set_ext(&g.tc, a2, b2, n_ext));
  g.split = S;
  if (S > 1) ws_floats_ = std::max<int64_t>(ws_floats_, S * M * N);
  return TTT_OK;
}

template <typename T>
int Engine<T>::run(Gemm& g, int64_t rows) {
  GemmShape s = g.shape;
  if (rows > 0 && !s.a_mn) s.a.rows = rows;
  const double flops = g.recompute ? 0.0 : 2.0 * (double)s.M() * (double)s.N() * (double)s.K();
  if (BF) {
    TcGemm tc = g.tc;
    tc.args = g.args;
    if (rows > 0 && !tc.a_mn) tc.M = rows;
    return timed(TTT_KC_GEMM, flops, [&] { return tc_gemm_launch(tc, st_, err_); }, g.label);
  }
  return timed(TTT_KC_GEMM, flops, [&] { return simt_gemm(s, g.epi, g.args, st_); }, g.label);
}

template <typename T>
int Engine<T>::init() {
  L_ = cfg_.n_layers;
  d_ = cfg_.d_model;
  f_ = cfg_.d_ff;
  H_ = cfg_.n_heads;
  HD_ = cfg_.head_dim;
  V_ = cfg_.vocab;
  nbot_ = L_ - nu_;
  scale_ = 1.f / std::sqrt((float)HD_);
  const int64_t d = d_, f = f_, b = b_;
  arena_.stream = st_;
  if (const char* t = getenv("TTT_TRACE")) {
    trace_ = t[0] && t[0] != '0';
    trace_verbose_ = t[0] == 'v';
    trace_ms_ = (float)atof(t) > 1.f ? (float)atof(t) : 0.f;  // TTT_TRACE=<ms>: log launches slower than that
  }
  if (const char* t = getenv("TTT_PROFILE")) timer_.labels = t[0] && t[0] != '0';
  TRY(arena_.alloc(&err_, 1));

  // Super-chunk length for the fast-weight-free blocks: about 16K positions.
  int64_t spc = std::max<int64_t>(1, 16384 / b);
  S_ = spc * b;
  // ring slots: at least window + chunk - 1, a multiple of 128 (key tiles of the
  // tensor-core attention start on 128-aligned positions)
  R1_ = (S_ + k_ + 127) / 128 * 128;
  R_ = (k_ + b + 127) / 128 * 128;

  // ---- weights ----------------------------------------------------------------------------
  wqkv_.resize(L_);
  wgu_.resize(L_);
  wd_.resize(L_);
  for (int64_t l = 0; l < L_; ++l) {
    const ttt_layer_weights& lw = wt_.layers[l];
    TRY(arena_.alloc(&wqkv_[l], 3 * d * d));
    TTT_CUDA_TRY(cudaMemcpyAsync(wqkv_[l], lw.wq, d * d * sizeof(T), cudaMemcpyDeviceToDevice, st_));
    TTT_CUDA_TRY(cudaMemcpyAsync(wqkv_[l] + d * d, lw.wk, d * d * sizeof(T), cudaMemcpyDeviceToDevice, st_));
    TTT_CUDA_TRY(cudaMemcpyAsync(wqkv_[l] + 2 * d * d, lw.wv, d * d * sizeof(T), cudaMemcpyDeviceToDevice, st_));
  }
  // gate/up rows interleaved in (gate 64 | up 64) blocks; the top blocks append the fast half
  m_gu_.assign(nu_, nullptr);
  m_d_.assign(nu_, nullptr);
  gu_lo_.assign(nu_, nullptr);
  d_lo_.assign(nu_, nullptr);
  init_gu_.assign(nu_, nullptr);
  init_d_.assign(nu_, nullptr);
  for (int64_t l = 0; l < L_; ++l) {
    const ttt_layer_weights& lw = wt_.layers[l];
    const bool top = l >= nbot_;
    TRY(arena_.alloc(&wgu_[l], (top ? 4 : 2) * f * d));
    TRY((interleave_gate_up<T, T>(reinterpret_cast<const T*>(lw.w_gate), reinterpret_cast<const T*>(lw.w_up), (int)f,
                                 (int)d, wgu_[l], st_)));
    if (top) {
      const int64_t i = l - nbot_;
      const ttt_fast_weights& fw = wt_.fast[i];
      TRY(arena_.alloc(&init_gu_[i], 2 * f * d));
      TRY(arena_.alloc(&init_d_[i], d * f));
      TRY((interleave_gate_up<float, float>(fw.w_gate, fw.w_up, (int)f, (int)d, init_gu_[i], st_)));
      TTT_CUDA_TRY(cudaMemcpyAsync(init_d_[i], fw.w_down, d * f * sizeof(float), cudaMemcpyDeviceToDevice, st_));
      TRY(arena_.alloc(&wd_[l], d * 2 * f));
      TRY(copy2d<T>(reinterpret_cast<const T*>(lw.w_down), f, wd_[l], 2 * f, d, f, st_));
      if (BF) {
        TRY(arena_.alloc(&m_gu_[i], 2 * f * d));
        TRY(arena_.alloc(&m_d_[i], d * f));
        TRY(arena_.alloc(&gu_lo_[i], 2 * f * d));
        TRY(arena_.alloc(&d_lo_[i], d * f));
      }
    } else {
      wd_[l] = const_cast<T*>(reinterpret_cast<const T*>(lw.w_down));
    }
  }
  TRY(reset());

  // ---- activations ------------------------------------------------------------------------
  if (nbot_ > 0) {
    TRY(arena_.alloc(&hs_, S_ * d));
    TRY(arena_.alloc(&qkvs_, S_ * 3 * d));
    TRY(arena_.alloc(&qs_, S_ * d));
    TRY(arena_.alloc(&os_, S_ * d));
    TRY(arena_.alloc(&as_, S_ * f));
    TRY(arena_.alloc(&rs_, S_));
    TRY(arena_.alloc(&rqs_, S_ * H_));
    TRY(arena_.alloc(&rks_, S_ * H_));
    TRY(arena_.alloc(&lses_, H_ * S_));
    kb_.resize(nbot_);
    vb_.resize(nbot_);
    for (int64_t l = 0; l < nbot_; ++l) {
      TRY(arena_.alloc(&kb_[l], R1_ * d));
      TRY(arena_.alloc(&vb_[l], R1_ * d));
    }
  }
  TRY(arena_.alloc(&xs_, S_ * d));
  TRY(arena_.alloc(&rope_tab_, S_ * (HD_ / 2)));
  auto per = [&](auto& vec) { vec.assign(nu_, nullptr); };
  per(xin_); per(r1_); per(xmid_); per(r2_); per(rq_); per(rk_); per(lse_);
  per(h_); per(qkv_); per(q_); per(o_); per(h2_); per(gu_); per(a_); per(kt_); per(vt_);
  for (int i = 0; i < nu_; ++i) {
    if (i > 0) TRY(arena_.alloc(&xin_[i], b * d));  // xin_[0] points into xs_
    TRY(arena_.alloc(&r1_[i], b));
    TRY(arena_.alloc(&xmid_[i], b * d));
    TRY(arena_.alloc(&r2_[i], b));
    TRY(arena_.alloc(&rq_[i], b * H_));
    TRY(arena_.alloc(&rk_[i], b * H_));
    TRY(arena_.alloc(&lse_[i], H_ * b));
    TRY(arena_.alloc(&h_[i], b * d));
    TRY(arena_.alloc(&qkv_[i], b * 3 * d));
    TRY(arena_.alloc(&q_[i], b * d));
    TRY(arena_.alloc(&o_[i], b * d));
    TRY(arena_.alloc(&h2_[i], b * d));
    TRY(arena_.alloc(&gu_[i], b * 4 * f));
    TRY(arena_.alloc(&a_[i], b * 2 * f));
    TRY(arena_.alloc(&kt_[i], R_ * d));
    TRY(arena_.alloc(&vt_[i], R_ * d));
  }
  TRY(arena_.alloc(&xf_, b * d));
  TRY(arena_.alloc(&rf_, b));
  TRY(arena_.alloc(&hf_, b * d));
  ce_tiles_ = BF ? tc_ce_tiles(V_, tc_pick_bn(b, V_, 0)) : (V_ + 127) / 128;
  TRY(arena_.alloc(&pmax_, ce_tiles_ * b));
  TRY(arena_.alloc(&psum_, ce_tiles_ * b));
  TRY(arena_.alloc(&zt_, b));
  TRY(arena_.alloc(&lsef_, b));
  TRY(arena_.alloc(&scl_, b));
  TRY(arena_.alloc(&tgt_, b));
  TRY(arena_.alloc(&dx_, b * d));
  TRY(arena_.alloc(&dxm_, b * d));
  TRY(arena_.alloc(&dhf_, b * d));
  TRY(arena_.alloc(&dh2_, b * d));
  TRY(arena_.alloc(&dh_, b * d));
  TRY(arena_.alloc(&Dbuf_, H_ * b));
  TRY(arena_.alloc(&dx16_, b * d));
  TRY(arena_.alloc(&dxm16_, b * d));
  // vocab chunk of the LM-head backward: the dz chunk stays L2-sized (<= 48 MB)
  {
    const int64_t max_cols = std::max<int64_t>(256, (48ll << 20) / (b * (int64_t)sizeof(T)) / 256 * 256);
    nvc_ = (V_ + max_cols - 1) / max_cols;
    Vc_ = ((V_ + nvc_ - 1) / nvc_ + 255) / 256 * 256;
    nvc_ = (V_ + Vc_ - 1) / Vc_;
  }
  TRY(arena_.alloc(&dz_, b * Vc_));
  if (BF) TRY(arena_.alloc(&logits_, b * V_));
  TRY(arena_.alloc(&da_, b * 2 * f));
  TRY(arena_.alloc(&dgu_, b * 4 * f));
  TRY(arena_.alloc(&do_, b * d));
  TRY(arena_.alloc(&dqkv_, b * 3 * d));
  // generation
  TRY(arena_.alloc(&dtok_, 1));
  TRY(arena_.alloc(&dloss_, 1));
  TRY(arena_.alloc(&xd_, d));
  TRY(arena_.alloc(&adws_, attn_decode_ws_floats((int)H_, (int)HD_, k_)));
  gvparts_ = gemv_parts(V_);
  TRY(arena_.alloc(&gvpart_, 3 * gvparts_));

  // ---- attention plans ----------------------------------------------------------------------
  tc_attn_ = BF && swa_tc_supported((int)HD_);
  qn_max_.assign(L_, 0.f);
  kn_max_.assign(L_, 0.f);
  if (tc_attn_) {
    std::vector<float> gq(HD_), gk(HD_);
    for (int64_t l = 0; l < L_; ++l) {
      TTT_CUDA_TRY(cudaMemcpyAsync(gq.data(), wt_.layers[l].q_norm, HD_ * sizeof(float), cudaMemcpyDeviceToHost, st_));
      TTT_CUDA_TRY(cudaMemcpyAsync(gk.data(), wt_.layers[l].k_norm, HD_ * sizeof(float), cudaMemcpyDeviceToHost, st_));
      TTT_CUDA_TRY(cudaStreamSynchronize(st_));
      float mq = 0.f, mk = 0.f;
      for (int64_t c = 0; c < HD_; ++c) {
        mq = std::max(mq, std::fabs(gq[c]));
        mk = std::max(mk, std::fabs(gk[c]));
      }
      // RMSNorm output rows have norm <= sqrt(head_dim) before the gain; RoPE keeps the norm
      if (std::isfinite(mq) && std::isfinite(mk)) {
        qn_max_[l] = mq * std::sqrt((float)HD_);
        kn_max_[l] = mk * std::sqrt((float)HD_);
      }
    }
  }
  if (tc_attn_) {
    att_bot_.resize(nbot_);
    att_top_.resize(nu_);
    for (int64_t l = 0; l < nbot_; ++l)
      TRY(swa_tc_prepare(&att_bot_[l], (int)H_, (int)HD_, qs_, S_, d, kb_[l], vb_[l], R1_, d));
    for (int i = 0; i < nu_; ++i)
      TRY(swa_tc_prepare(&att_top_[i], (int)H_, (int)HD_, q_[i], b, d, kt_[i], vt_[i], R_, d));
    att_bwd_.resize(nu_);
    for (int i = 1; i < nu_; ++i)
      TRY(swa_tc_bwd_prepare(&att_bwd_[i], (int)H_, (int)HD_, q_[i], do_, b, d, kt_[i], vt_[i], R_, d));
  }

  // ---- GEMM plans -------------------------------------------------------------------------
  EpiArgs e;
  g_bot_.resize(4 * nbot_);
  for (int64_t l = 0; l < nbot_; ++l) {
    Gemm* g = &g_bot_[4 * l];
    e = EpiArgs{}; e.c = qkvs_; e.ldc = 3 * d;
    TRY(prep(g[0], 0, MatView{hs_, S_, d, d}, 0, MatView{wqkv_[l], 3 * d, d, d}, STORE, e));
    g[0].label = "bot.qkv";
    e = EpiArgs{}; e.c = xs_; e.ldc = d;
    TRY(prep(g[1], 0, MatView{os_, S_, d, d}, 0, MatView{wt_.layers[l].wo, d, d, d}, EPI_ADD_F32, e));
    g[1].label = "bot.o";
    e = EpiArgs{}; e.c = as_; e.ldc = f;
    TRY(prep(g[2], 0, MatView{hs_, S_, d, d}, 0, MatView{wgu_[l], 2 * f, d, d}, EPI_SWIGLU, e));
    g[2].label = "bot.gateup";
    e = EpiArgs{}; e.c = xs_; e.ldc = d;
    TRY(prep(g[3], 0, MatView{as_, S_, f, f}, 0, MatView{wd_[l], d, f, f}, EPI_ADD_F32, e));
    g[3].label = "bot.down";
  }
  g_top_.resize(10 * nu_);
  for (int i = 0; i < nu_; ++i) {
    const int64_t l = nbot_ + i;
    Gemm* g = &g_top_[10 * i];
    e = EpiArgs{}; e.c = qkv_[i]; e.ldc = 3 * d;
    TRY(prep(g[0], 0, MatView{h_[i], b, d, d}, 0, MatView{wqkv_[l], 3 * d, d, d}, STORE, e));
    g[0].label = "top.qkv";
    e = EpiArgs{}; e.c = xmid_[i]; e.ldc = d; e.ldc2 = d;  // c2 = x_in, set per chunk
    TRY(prep(g[1], 0, MatView{o_[i], b, d, d}, 0, MatView{wt_.layers[l].wo, d, d, d}, EPI_ADD_F32, e));
    g[1].label = "top.o";
    e = EpiArgs{}; e.c = a_[i]; e.ldc = 2 * f; e.c2 = gu_[i]; e.ldc2 = 4 * f;
    TRY(prep(g[2], 0, MatView{h2_[i], b, d, d}, 0, MatView{wgu_[l], 4 * f, d, d}, EPI_SWIGLU, e));
    g[2].label = "top.gateup";
    // fast half: + h2 W_lo^T
    TRY(prep_ext(g[2], MatView{h2_[i], b, d, d}, MatView{gu_lo_[i], 2 * f, d, d}, 2 * f));
    e = EpiArgs{}; e.c = (i + 1 < nu_) ? xin_[i + 1] : xf_; e.ldc = d; e.c2 = xmid_[i]; e.ldc2 = d;
    TRY(prep(g[3], 0, MatView{a_[i], b, 2 * f, 2 * f}, 0, MatView{wd_[l], d, 2 * f, 2 * f}, EPI_ADD_F32, e));
    g[3].label = "top.down";
    // + a_fast W_down,lo^T
    TRY(prep_ext(g[3], MatView{a_[i] + f, b, f, 2 * f}, MatView{d_lo_[i], d, f, f}, 0));
    // backward: da (fast half only in the lowest updated block)
    if (i == 0) {
      e = EpiArgs{}; e.c = da_ + f; e.ldc = 2 * f;
      TRY(prep(g[4], 0, MatView{dx16_, b, d, d}, 1, MatView{wd_[l] + f, d, f, 2 * f}, STORE, e));
      g[4].label = "top.da";
    } else {
      e = EpiArgs{}; e.c = da_; e.ldc = 2 * f;
      TRY(prep(g[4], 0, MatView{dx16_, b, d, d}, 1, MatView{wd_[l], d, 2 * f, 2 * f}, STORE, e));
      g[4].label = "top.da";
      e = EpiArgs{}; e.c = dh2_; e.ldc = d;
      TRY(prep(g[5], 0, MatView{dgu_, b, 4 * f, 4 * f}, 1, MatView{wgu_[l], 4 * f, d, d}, EPI_STORE_F32, e));
      g[5].label = "top.dgrad_gu";
    }
    // weight gradients + SGD on the fast halves
    e = EpiArgs{}; e.alpha = eta_;
    if (BF) { e.c = m_d_[i]; e.ldc = f; e.c2 = wd_[l] + f; e.ldc2 = 2 * f; e.c3 = d_lo_[i]; e.ldc3 = f; }
    else { e.c = wd_[l] + f; e.ldc = 2 * f; }
    TRY(prep(g[6], 1, MatView{dx16_, b, d, d}, 1, MatView{a_[i] + f, b, f, 2 * f}, EPI_SGD, e));
    g[6].label = "top.sgd_down";
    e = EpiArgs{}; e.alpha = eta_;
    if (BF) { e.c = m_gu_[i]; e.ldc = d; e.c2 = wgu_[l] + 2 * f * d; e.ldc2 = d; e.c3 = gu_lo_[i]; e.ldc3 = d; }
    else { e.c = wgu_[l] + 2 * f * d; e.ldc = d; }
    TRY(prep(g[7], 1, MatView{dgu_ + 2 * f, b, 2 * f, 4 * f}, 1, MatView{h2_[i], b, d, d}, EPI_SGD, e));
    g[7].label = "top.sgd_gu";
    if (i > 0) {
      e = EpiArgs{}; e.c = do_; e.ldc = d;
      TRY(prep(g[8], 0, MatView{dxm16_, b, d, d}, 1, MatView{wt_.layers[l].wo, d, d, d}, STORE, e));
      g[8].label = "top.dgrad_o";
      e = EpiArgs{}; e.c = dh_; e.ldc = d;
      TRY(prep(g[9], 0, MatView{dqkv_, b, 3 * d, 3 * d}, 1, MatView{wqkv_[l], 3 * d, d, d}, EPI_STORE_F32, e));
      g[9].label = "top.dgrad_qkv";
    }
  }
  e = EpiArgs{}; e.row_i = tgt_; e.part_max = pmax_; e.part_sum = psum_; e.target_logit = zt_; e.part_ld = b;
  if (BF) { e.c = logits_; e.ldc = V_; }  // the logits stay for the backward
  TRY(prep(g_head_, 0, MatView{hf_, b, d, d}, 0, MatView{wt_.lm_head, V_, d, d}, EPI_CE_FWD, e));
  g_head_.label = "head.ce_fwd";
  g_ce_dz_.resize(nvc_);
  g_ce_dh_.resize(nvc_);
  for (int64_t c = 0; c < nvc_; ++c) {
    const int64_t v0 = c * Vc_, vn = std::min<int64_t>(Vc_, V_ - v0);
    const T* hv = reinterpret_cast<const T*>(wt_.lm_head) + v0 * d;
    e = EpiArgs{}; e.c = dz_; e.ldc = Vc_; e.row_f = lsef_; e.row_g = scl_; e.row_i = tgt_; e.col_offset = v0;
    TRY(prep(g_ce_dz_[c], 0, MatView{hf_, b, d, d}, 0, MatView{hv, vn, d, d}, EPI_CE_BWD, e));
    g_ce_dz_[c].label = "head.ce_dz";
    g_ce_dz_[c].recompute = true;
    e = EpiArgs{}; e.c = dhf_; e.ldc = d;
    TRY(prep(g_ce_dh_[c], 0, MatView{dz_, b, vn, Vc_}, 1, MatView{hv, vn, d, d}, c == 0 ? EPI_STORE_F32 : EPI_ADD_F32,
             e));
    g_ce_dh_[c].label = "head.ce_dh";
  }
  TRY(finalize_splits());
  TTT_CUDA_TRY(cudaStreamSynchronize(st_));
  return TTT_OK;
}


template <typename T>
int Engine<T>::reset() {
  const int64_t d = d_, f = f_;
  for (int i = 0; i < nu_; ++i) {
    const int64_t l = nbot_ + i;
    timer_.cut();
    TTT_CUDA_TRY(cudaMemcpyAsync(master_gu(i), init_gu_[i], 2 * f * d * sizeof(float), cudaMemcpyDeviceToDevice, st_));
    TRY(timed(TTT_KC_OTHER, 0, [&] { return copy2d<float>(init_d_[i], f, master_d(i), master_d_ld(), d, f, st_); }));
    if (BF) {
      TRY(timed(TTT_KC_OTHER, 0, [&] { return copy2d_from_f32<T>(init_gu_[i], d, wgu_[l] + 2 * f * d, d, 2 * f, d, st_); }));
      TRY(timed(TTT_KC_OTHER, 0, [&] { return copy2d_from_f32<T>(init_d_[i], f, wd_[l] + f, 2 * f, d, f, st_); }));
      TRY(timed(TTT_KC_OTHER, 0, [&] { return bf16_lo2d(init_gu_[i], d, gu_lo_[i], d, 2 * f, d, st_); }));
      TRY(timed(TTT_KC_OTHER, 0, [&] { return bf16_lo2d(init_d_[i], f, d_lo_[i], f, d, f, st_); }));
    }
  }
  fresh_ = true;
  prefilled_ = dec_ready_ = false;
  dec_pos_ = 0;
  return TTT_OK;
}

template <typename T>
int Engine<T>::sync() {
  TTT_CUDA_TRY(cudaStreamSynchronize(st_));
  int h = 0;
  TTT_CUDA_TRY(cudaMemcpy(&h, err_, sizeof(int), cudaMemcpyDeviceToHost));
  if (h) {
    TTT_CUDA_TRY(cudaMemset(err_, 0, sizeof(int)));
    TTT_CUDA_TRY(cudaDeviceSynchronize());
    if (h & DEV_ERR_BAD_TOKEN) return set_error(TTT_ERR_INVALID_ARG, "a token id lies outside [0, vocab)");
    return set_error(TTT_ERR_TIMEOUT, "a kernel's bounded wait timed out (device watchdog)");
  }
  return TTT_OK;
}

template <typename T>
int Engine<T>::bottom_layers(const int32_t* tok, int64_t s0, int64_t S) {
  phase_ = "bot";
  const int64_t d = d_;
  const float eps = cfg_.norm_eps;
  const double theta = cfg_.rope_theta;
  TRY(timed(TTT_KC_OTHER, 0, [&] { return embed_gather<T>(tok + s0, reinterpret_cast<const T*>(wt_.embed), S, (int)d, (int)V_, xs_, err_, st_); }));
  // rotation table of this super-chunk's positions: every block and chunk inside it reads it
  tab_p0_ = s0;
  TRY(timed(TTT_KC_ROPE, 0, [&] { return rope_table(rope_tab_, s0, S, (int)HD_, theta, st_); }));
  for (int64_t l = 0; l < nbot_; ++l) {
    const ttt_layer_weights& lw = wt_.layers[l];
    Gemm* g = &g_bot_[4 * l];
    TRY(timed(TTT_KC_NORM, 0, [&] { return rmsnorm_fwd<T>(xs_, d, lw.attn_norm, eps, S, (int)d, hs_, d, rs_, st_); }));
    TRY(run(g[0], S));
    TRY(timed(TTT_KC_ROPE, 0, [&] { return qknorm_rope_fwd<T>(qkvs_, 3 * d, lw.q_norm, lw.k_norm, S, s0, (int)H_, (int)HD_, eps, rope_tab_, tab_p0_, qs_, d,
                                 kb_[l], vb_[l], d, R1_, rqs_, rks_, st_); }));
    TRY(timed(TTT_KC_ATTN_FWD, 4.0 * d * band_pairs(s0, S),
              [&] { return attn_fwd(tc_attn_ ? &att_bot_[l] : nullptr,
                                    swa_args(qs_, S, s0, kb_[l], vb_[l], R1_, os_, lses_, S_, l)); }));
    TRY(run(g[1], S));
    TRY(timed(TTT_KC_NORM, 0, [&] { return rmsnorm_fwd<T>(xs_, d, lw.mlp_norm, eps, S, (int)d, hs_, d, rs_, st_); }));
    TRY(run(g[2], S));
    TRY(run(g[3], S));
  }
  return TTT_OK;
}

template <typename T>
int Engine<T>::chunk(const int32_t* tok, int64_t T_, int64_t p0, int64_t n, const float* x0, float* losses) {
  phase_ = "top";
  const int64_t d = d_, f = f_, b = b_;
  const float eps = cfg_.norm_eps;
  const double theta = cfg_.rope_theta;
  const int64_t n_valid = std::max<int64_t>(0, std::min<int64_t>(n, T_ - 1 - p0));
  TRY(timed(TTT_KC_OTHER, 0, [&] { return chunk_targets(tok, T_, p0, n, tgt_, st_); }));
  // ---- forward of the updated blocks with the current fast weights ----
  for (int i = 0; i < nu_; ++i) {
    const int64_t l = nbot_ + i;
    const ttt_layer_weights& lw = wt_.layers[l];
    Gemm* g = &g_top_[10 * i];
    const float* xin = i == 0 ? x0 : xin_[i];
    TRY(timed(TTT_KC_NORM, 0, [&] { return rmsnorm_fwd<T>(xin, d, lw.attn_norm, eps, n, (int)d, h_[i], d, r1_[i], st_); }));
    TRY(run(g[0], n));
    TRY(timed(TTT_KC_ROPE, 0, [&] { return qknorm_rope_fwd<T>(qkv_[i], 3 * d, lw.q_norm, lw.k_norm, n, p0, (int)H_, (int)HD_, eps, rope_tab_, tab_p0_, q_[i], d,
                                 kt_[i], vt_[i], d, R_, rq_[i], rk_[i], st_); }));
    TRY(timed(TTT_KC_ATTN_FWD, 4.0 * d * band_pairs(p0, n),
              [&] { return attn_fwd(tc_attn_ ? &att_top_[i] : nullptr,
                                    swa_args(q_[i], n, p0, kt_[i], vt_[i], R_, o_[i], lse_[i], b, l)); }));
    g[1].args.c2 = const_cast<float*>(xin);
    TRY(run(g[1], n));
    TRY(timed(TTT_KC_NORM, 0, [&] { return rmsnorm_fwd<T>(xmid_[i], d, lw.mlp_norm, eps, n, (int)d, h2_[i], d, r2_[i], st_); }));
    TRY(run(g[2], n));
    TRY(run(g[3], n));
  }
  TRY(timed(TTT_KC_NORM, 0, [&] { return rmsnorm_fwd<T>(xf_, d, wt_.final_norm, eps, n, (int)d, hf_, d, rf_, st_); }));
  TRY(run(g_head_, n));
  TRY(timed(TTT_KC_OTHER, 0, [&] { return ce_finalize(pmax_, psum_, b, (int)ce_tiles_, zt_, n, n_valid, n_valid ? 1.f / (float)n_valid : 0.f,
                        losses + p0, lsef_, scl_, st_); }));
  if (n < b || n_valid == 0) return TTT_OK;  // a trailing partial chunk is scored only
  // eta = 0: the step W -= 0 * G leaves every weight as it is, so the
  // backward that would produce G is skipped (the L_static model of eq. (4))
  if (eta_ == 0.f) return TTT_OK;
  return chunk_backward(p0, n, BF);
}

template <typename T>
int Engine<T>::chunk_backward(int64_t p0, int64_t n, bool logits_stored) {
  const int64_t d = d_, f = f_, b = b_;
  // ---- backward through the updated blocks, SGD on each fast MLP ----
  phase_ = "bwd";
  for (int64_t c = 0; c < nvc_; ++c) {
    const int64_t v0 = c * Vc_, vn = std::min<int64_t>(Vc_, V_ - v0);
    if (logits_stored)  // dz of this vocab chunk from the forward's logits (L2-sized, read by the next product)
      TRY(timed(TTT_KC_OTHER, 0, [&] { return ce_grad_from_logits<T>(logits_, V_, lsef_, scl_, tgt_, v0, n, vn, dz_, Vc_, st_); }, "head.ce_grad"));
    else
      TRY(run(g_ce_dz_[c], n));
    TRY(run(g_ce_dh_[c], n));
  }
  TRY(timed(TTT_KC_NORM, 0, [&] { return rmsnorm_bwd<T>(xf_, d, rf_, wt_.final_norm, dhf_, d, nullptr, 0, n, (int)d, dx_, d, dx16_, d, st_); }));
  for (int i = nu_ - 1; i >= 0; --i) {
    const int64_t l = nbot_ + i;
    const ttt_layer_weights& lw = wt_.layers[l];
    Gemm* g = &g_top_[10 * i];
    TRY(run(g[4], n));
    if (i == 0) {
      TRY(timed(TTT_KC_OTHER, 0, [&] { return swiglu_bwd<T>(da_ + f, 2 * f, gu_[i] + 2 * f, 4 * f, n, f, dgu_ + 2 * f, 4 * f, st_); }));
    } else {
      TRY(timed(TTT_KC_OTHER, 0, [&] { return swiglu_bwd<T>(da_, 2 * f, gu_[i], 4 * f, n, 2 * f, dgu_, 4 * f, st_); }));
      TRY(run(g[5], n));  // reads the fast shadow before its update
    }
    TRY(run(g[6], 0));  // W_down fast -= eta * dx^T a_f
    TRY(run(g[7], 0));  // W_gate/up fast -= eta * dgu_f^T h2
    if (i == 0) break;  // nothing below the lowest fast block depends on W
    TRY(timed(TTT_KC_NORM, 0, [&] { return rmsnorm_bwd<T>(xmid_[i], d, r2_[i], lw.mlp_norm, dh2_, d, dx_, d, n, (int)d, dxm_, d, dxm16_, d, st_); }));
    TRY(run(g[8], n));
    SwaArgs a = swa_args(q_[i], n, p0, kt_[i], vt_[i], R_, o_[i], lse_[i], b, l);
    a.dout = do_;
    a.lddo = d;
    a.dq = dqkv_;
    a.lddq = 3 * d;
    a.dk = dqkv_ + d;
    a.dv = dqkv_ + 2 * d;
    a.lddkv = 3 * d;
    a.D = Dbuf_;
    TRY(timed(TTT_KC_ATTN_BWD, 4.0 * d * (band_pairs(p0, n) + (double)n * (double)(n + 1) / 2.0), [&] {
      if (tc_attn_) {
        std::function<int()> dkdv;
        if (swa_tc_dkdv_supported(a)) dkdv = [&] { return swa_tc_backward_dkdv(att_bwd_[i], a, st_, err_); };
        return swa_backward_with_dq(a, true, st_, [&] { return swa_tc_backward_dq(att_bwd_[i], a, st_, err_); },
                                    dkdv);
      }
      return swa_backward(a, BF, st_);
    }));
    launches += 2;  // the backward launches three kernels
    TRY(timed(TTT_KC_ROPE, 0, [&] { return qknorm_rope_bwd<T>(dqkv_, 3 * d, qkv_[i], 3 * d, lw.q_norm, lw.k_norm, rq_[i], rk_[i], n, p0, (int)H_,
                                 (int)HD_, rope_tab_, tab_p0_, st_); }));
    TRY(run(g[9], n));
    TRY(timed(TTT_KC_NORM, 0, [&] { return rmsnorm_bwd<T>(xin_[i], d, r1_[i], lw.attn_norm, dh_, d, dxm_, d, n, (int)d, dx_, d, dx16_, d, st_); }));
  }
  return TTT_OK;
}

template <typename T>
int Engine<T>::prefill(const int32_t* tok, int64_t T_, float* losses, float* const* fast_out) {
  if (!fresh_) return set_error(TTT_ERR_STATE, "ttt_prefill needs a fresh context (call ttt_reset)");
  if (!tok || !losses || T_ < 1) return set_error(TTT_ERR_INVALID_ARG, "ttt_prefill: bad argument");
  fresh_ = false;
  phase_ = "misc";
  timer_.cut();  // the caller may have enqueued work on the stream since the last call
  TRY(timed(TTT_KC_OTHER, 0, [&] { return check_tokens(tok, T_, (int)V_, err_, st_); }));
  for (int64_t s0 = 0; s0 < T_; s0 += S_) {
    const int64_t S = std::min<int64_t>(S_, T_ - s0);
    TRY(bottom_layers(tok, s0, S));
    for (int64_t p0 = s0; p0 < s0 + S; p0 += b_) {
      const int64_t n = std::min<int64_t>(b_, T_ - p0);
      TRY(chunk(tok, T_, p0, n, xs_ + (p0 - s0) * d_, losses));
    }
  }
  prefilled_ = true;
  dec_ready_ = false;
  dec_pos_ = T_;
  if (fast_out) {
    const int64_t d = d_, f = f_;
    for (int i = 0; i < nu_; ++i) {
      float* og = fast_out[3 * i];
      float* ou = fast_out[3 * i + 1];
      float* od = fast_out[3 * i + 2];
      if (!og || !ou || !od) return set_error(TTT_ERR_INVALID_ARG, "ttt_prefill: NULL entry in fast_out");
      TRY(timed(TTT_KC_OTHER, 0, [&] { return deinterleave_gate_up(master_gu(i), (int)f, (int)d, og, ou, st_); }));
      TRY(timed(TTT_KC_OTHER, 0, [&] { return copy2d<float>(master_d(i), master_d_ld(), od, f, d, f, st_); }));
    }
  }
  return TTT_OK;
}

template <typename T>
template <typename G>
int Engine<T>::gemv_run(const GemvArgs<T>& a, int epi, G&& label) {
  const double bytes = (double)sizeof(T) * ((double)a.n * (double)a.k + (a.w2 ? (double)(a.n - std::min<int64_t>(a.n, a.n_ext)) * (double)a.k2 : 0.0));
  return timed(TTT_KC_DECODE, bytes, [&] { return gemv<T>(a, epi, st_); }, label);
}

template <typename T>
int Engine<T>::head_pick(const T* hf, const float* xres, T* h_out, float* r_out, int32_t* tgt_row, float* lse_row) {
  GemvArgs<T> g;
  g.w = reinterpret_cast<const T*>(wt_.lm_head);
  g.ldw = d_;
  g.n = V_;
  g.k = d_;
  g.x = hf;
  if (!hf) {
    g.xres = xres;
    g.gain = wt_.final_norm;
    g.eps = cfg_.norm_eps;
    g.h_out = h_out;
    g.r_out = r_out;
  }
  g.out = gvpart_;  // unused by the argmax epilogue, must be non-NULL
  g.part = gvpart_;
  TRY(gemv_run(g, GEMV_ARGMAX, "dec.head"));
  return timed(TTT_KC_DECODE, 0, [&] { return argmax_finalize(gvpart_, gvparts_, dtok_, tgt_row, lse_row, dloss_, st_); },
               "dec.pick");
}

template <typename T>
int Engine<T>::decode_position(int64_t p) {
  const int64_t d = d_, f = f_, b = b_;
  const float eps = cfg_.norm_eps;
  const int64_t c0 = p - p % b, r = p - c0;
  phase_ = "dec";
  if (tab_p0_ != c0) {  // rotation table of this chunk's positions (also read by its backward)
    tab_p0_ = c0;
    TRY(timed(TTT_KC_DECODE, 0, [&] { return rope_table(rope_tab_, c0, b, (int)HD_, cfg_.rope_theta, st_); }, "dec.rope_table"));
  }
  TRY(timed(TTT_KC_DECODE, 0, [&] { return embed_gather<T>(dtok_, reinterpret_cast<const T*>(wt_.embed), 1, (int)d, (int)V_, xd_, err_, st_); }, "dec.embed"));
  const double kv_bytes = 2.0 * (double)sizeof(T) * (double)d * (double)std::min<int64_t>(p + 1, k_);
  // ---- blocks without fast weights: one row, scratch of the super-chunk buffers ----
  // (the RMSNorms run as the prologue of the product that reads them)
  for (int64_t l = 0; l < nbot_; ++l) {
    const ttt_layer_weights& lw = wt_.layers[l];
    GemvArgs<T> g;
    g.w = wqkv_[l]; g.ldw = d; g.n = 3 * d; g.k = d; g.out = qkvs_;
    g.xres = xd_; g.gain = lw.attn_norm; g.eps = eps;
    TRY(gemv_run(g, GEMV_STORE, "dec.qkv"));
    TRY(timed(TTT_KC_DECODE, 0, [&] { return qknorm_rope_fwd<T>(qkvs_, 3 * d, lw.q_norm, lw.k_norm, 1, p, (int)H_, (int)HD_, eps, rope_tab_, tab_p0_, qs_, d, kb_[l], vb_[l], d, R1_, rqs_, rks_, st_); }, "dec.qknorm_rope"));
    TRY(timed(TTT_KC_DECODE, kv_bytes, [&] { return attn_decode<T>(qs_, kb_[l], vb_[l], d, R1_, (int)H_, (int)HD_, p, k_, scale_, os_, nullptr, 0, adws_, st_); }, "dec.attn"));
    g = GemvArgs<T>();
    g.w = reinterpret_cast<const T*>(lw.wo); g.ldw = d; g.n = d; g.k = d; g.x = os_; g.out = xd_; g.res = xd_;
    TRY(gemv_run(g, GEMV_ADD_F32, "dec.o"));
    g = GemvArgs<T>();
    g.w = wgu_[l]; g.ldw = d; g.n = 2 * f; g.k = d; g.out = as_;
    g.xres = xd_; g.gain = lw.mlp_norm; g.eps = eps;
    TRY(gemv_run(g, GEMV_SWIGLU, "dec.gateup"));
    g = GemvArgs<T>();
    g.w = wd_[l]; g.ldw = f; g.n = d; g.k = f; g.x = as_; g.out = xd_; g.res = xd_;
    TRY(gemv_run(g, GEMV_ADD_F32, "dec.down"));
  }
  // ---- blocks with fast weights: row r of the chunk buffers (the chunk's backward reads them) ----
  for (int i = 0; i < nu_; ++i) {
    const int64_t l = nbot_ + i;
    const ttt_layer_weights& lw = wt_.layers[l];
    const float* xin = i == 0 ? xd_ : xin_[i] + r * d;
    T* h = h_[i] + r * d;
    T* qkv = qkv_[i] + r * 3 * d;
    T* q = q_[i] + r * d;
    T* o = o_[i] + r * d;
    T* h2 = h2_[i] + r * d;
    T* a = a_[i] + r * 2 * f;
    float* xmid = xmid_[i] + r * d;
    float* xout = (i + 1 < nu_ ? xin_[i + 1] : xf_) + r * d;
    GemvArgs<T> g;
    g.w = wqkv_[l]; g.ldw = d; g.n = 3 * d; g.k = d; g.out = qkv;
    g.xres = xin; g.gain = lw.attn_norm; g.eps = eps; g.h_out = h; g.r_out = r1_[i] + r;
    TRY(gemv_run(g, GEMV_STORE, "dec.qkv"));
    TRY(timed(TTT_KC_DECODE, 0, [&] { return qknorm_rope_fwd<T>(qkv, 3 * d, lw.q_norm, lw.k_norm, 1, p, (int)H_, (int)HD_, eps, rope_tab_, tab_p0_, q, d, kt_[i], vt_[i], d, R_, rq_[i] + r * H_, rk_[i] + r * H_, st_); }, "dec.qknorm_rope"));
    TRY(timed(TTT_KC_DECODE, kv_bytes, [&] { return attn_decode<T>(q, kt_[i], vt_[i], d, R_, (int)H_, (int)HD_, p, k_, scale_, o, lse_[i] + r, b, adws_, st_); }, "dec.attn"));
    g = GemvArgs<T>();
    g.w = reinterpret_cast<const T*>(lw.wo); g.ldw = d; g.n = d; g.k = d; g.x = o; g.out = xmid; g.res = xin;
    TRY(gemv_run(g, GEMV_ADD_F32, "dec.o"));
    // [static | fast] gate/up with the SwiGLU epilogue; bf16: + h2 W_lo^T on the fast rows
    g = GemvArgs<T>();
    g.w = wgu_[l]; g.ldw = d; g.n = 4 * f; g.k = d; g.out = a; g.raw = gu_[i] + r * 4 * f;
    g.xres = xmid; g.gain = lw.mlp_norm; g.eps = eps; g.h_out = h2; g.r_out = r2_[i] + r;
    if (BF) { g.w2 = reinterpret_cast<const T*>(gu_lo_[i]); g.ldw2 = d; g.k2 = d; g.n_ext = 2 * f; }
    TRY(gemv_run(g, GEMV_SWIGLU, "dec.gateup"));
    // [static | fast] down + residual; bf16: + a_fast W_down,lo^T
    g = GemvArgs<T>();
    g.w = wd_[l]; g.ldw = 2 * f; g.n = d; g.k = 2 * f; g.x = a; g.out = xout; g.res = xmid;
    if (BF) { g.w2 = reinterpret_cast<const T*>(d_lo_[i]); g.ldw2 = f; g.k2 = f; g.x2 = a + f; g.n_ext = 0; }
    TRY(gemv_run(g, GEMV_ADD_F32, "dec.down"));
  }
  // next token = greedy pick of this position's logits (final RMSNorm in the
  // product's prologue); it is also this row's target
  TRY(head_pick(nullptr, xf_ + r * d, hf_ + r * d, rf_ + r, tgt_ + r, lsef_ + r));
  if (r == b - 1 && eta_ != 0.f) {
    // the chunk [c0, c0 + b) is complete: every position has its target
    TRY(timed(TTT_KC_DECODE, 0, [&] { return fill_f32(scl_, b, 1.f / (float)b, st_); }, "dec.scale"));
    TRY(chunk_backward(c0, b, false));  // decode positions kept no logits: recompute them
  }
  return TTT_OK;
}

template <typename T>
int Engine<T>::decode(int64_t count, int32_t* tokens, float* losses) {
  if (!prefilled_) return set_error(TTT_ERR_STATE, "ttt_decode needs a ttt_prefill of the prompt first");
  if (count < 0 || (count > 0 && !tokens)) return set_error(TTT_ERR_INVALID_ARG, "ttt_decode: bad argument");
  timer_.cut();
  if (!dec_ready_) {
    // the token after the prompt comes from the logits of its last position,
    // scored with the weights of that position's chunk (the final-norm row
    // the prefill left in hf_)
    const int64_t p = dec_pos_ - 1, r = p % b_;
    phase_ = "dec";
    TRY(head_pick(hf_ + r * d_, nullptr, nullptr, nullptr, tgt_ + r, nullptr));
    dec_ready_ = true;
  }
  for (int64_t i = 0; i < count; ++i) {
    timer_.cut();
    TTT_CUDA_TRY(cudaMemcpyAsync(tokens + i, dtok_, sizeof(int32_t), cudaMemcpyDeviceToDevice, st_));
    if (losses) TTT_CUDA_TRY(cudaMemcpyAsync(losses + i, dloss_, sizeof(float), cudaMemcpyDeviceToDevice, st_));
    TRY(decode_position(dec_pos_));
    ++dec_pos_;
  }
  return TTT_OK;
}

}  // namespace
}  // namespace ttt

// ---- C ABI ----------------------------------------------------------------------------------------

using namespace ttt;

static int fail(ttt_ctx* ctx, int rc) {
  if (rc != TTT_OK && ctx) ctx->last_error = last_error_message();
  return rc;
}

extern "C" int ttt_init(const ttt_config* c, const ttt_weights* w, float eta, int32_t k, int32_t b, int32_t nu,
                        void* stream, ttt_ctx** out) {
  if (out) *out = nullptr;
  if (!c || !w || !out) return set_error(TTT_ERR_INVALID_ARG, "ttt_init: NULL argument");
  const bool hd_ok = c->head_dim == 32 || c->head_dim == 64 || c->head_dim == 80 || c->head_dim == 96 ||
                     c->head_dim == 128;
  if (c->n_layers < 1 || c->n_heads < 1 || c->d_model != c->n_heads * c->head_dim || c->d_model % 8 ||
      c->d_ff < 64 || c->d_ff % 64 || c->vocab < 1 || !(c->norm_eps > 0.f) || !(c->rope_theta > 0.f))
    return set_error(TTT_ERR_INVALID_ARG, "ttt_init: bad model configuration");
  if (!hd_ok) return set_error(TTT_ERR_UNSUPPORTED, "ttt_init: head_dim must be 32, 64, 80, 96 or 128");
  if (c->dtype != TTT_F32 && c->dtype != TTT_BF16) return set_error(TTT_ERR_INVALID_ARG, "ttt_init: bad dtype");
  if (!std::isfinite(eta) || k < 1 || b < 1 || nu < 1 || nu > c->n_layers)
    return set_error(TTT_ERR_INVALID_ARG, "ttt_init: need finite eta, k >= 1, b >= 1, 1 <= n_updated <= n_layers");
  if (!w->embed || !w->layers || !w->fast || !w->final_norm || !w->lm_head)
    return set_error(TTT_ERR_INVALID_ARG, "ttt_init: NULL weight pointer");
  for (int l = 0; l < c->n_layers; ++l) {
    const ttt_layer_weights& lw = w->layers[l];
    if (!lw.attn_norm || !lw.wq || !lw.wk || !lw.wv || !lw.wo || !lw.q_norm || !lw.k_norm || !lw.mlp_norm ||
        !lw.w_gate || !lw.w_up || !lw.w_down)
      return set_error(TTT_ERR_INVALID_ARG, "ttt_init: NULL weight pointer in block " + std::to_string(l));
  }
  for (int i = 0; i < nu; ++i)
    if (!w->fast[i].w_gate || !w->fast[i].w_up || !w->fast[i].w_down)
      return set_error(TTT_ERR_INVALID_ARG, "ttt_init: NULL fast weight pointer");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  std::unique_ptr<ttt_ctx> ctx;
  int rc;
  if (c->dtype == TTT_BF16) {
    auto* e = new Engine<bf16>(*c, *w, eta, k, b, nu, s);
    ctx.reset(e);
    rc = e->init();
  } else {
    auto* e = new Engine<float>(*c, *w, eta, k, b, nu, s);
    ctx.reset(e);
    rc = e->init();
  }
  if (rc != TTT_OK) return rc;
  *out = ctx.release();
  return TTT_OK;
}

extern "C" int ttt_prefill(ttt_ctx* ctx, const int32_t* tokens_dev, int64_t T, float* losses_dev,
                           float* const* fast_out_dev) {
  if (!ctx) return set_error(TTT_ERR_INVALID_ARG, "ttt_prefill: NULL context");
  return fail(ctx, ctx->prefill(tokens_dev, T, losses_dev, fast_out_dev));
}

extern "C" int ttt_decode_step(ttt_ctx* ctx, int32_t* next_token_dev) {
  if (!ctx) return set_error(TTT_ERR_INVALID_ARG, "ttt_decode_step: NULL context");
  return fail(ctx, ctx->decode(1, next_token_dev, nullptr));
}

extern "C" int ttt_decode(ttt_ctx* ctx, int64_t n_tokens, int32_t* tokens_dev, float* losses_dev) {
  if (!ctx) return set_error(TTT_ERR_INVALID_ARG, "ttt_decode: NULL context");
  return fail(ctx, ctx->decode(n_tokens, tokens_dev, losses_dev));
}

extern "C" int ttt_reset(ttt_ctx* ctx) {
  if (!ctx) return set_error(TTT_ERR_INVALID_ARG, "ttt_reset: NULL context");
  return fail(ctx, ctx->reset());
}

extern "C" int ttt_sync(ttt_ctx* ctx) {
  if (!ctx) return set_error(TTT_ERR_INVALID_ARG, "ttt_sync: NULL context");
  return fail(ctx, ctx->sync());
}

extern "C" const char* ttt_last_error(ttt_ctx* ctx) {
  return ctx ? ctx->last_error.c_str() : last_error_message();
}

extern "C" void ttt_free(ttt_ctx* ctx) {
  if (!ctx) return;
  ctx->sync();
  delete ctx;
}

extern "C" int64_t ttt_launch_count(ttt_ctx* ctx) { return ctx ? ctx->launches : 0; }

extern "C" int ttt_timing_enable(ttt_ctx* ctx, int32_t enable) {
  if (!ctx) return set_error(TTT_ERR_INVALID_ARG, "ttt_timing_enable: NULL context");
  return fail(ctx, ctx->timing_enable(enable != 0));
}

extern "C" int ttt_timing_read(ttt_ctx* ctx, int32_t kc, double* total_ms, int64_t* launches, double* flops) {
  if (!ctx) return set_error(TTT_ERR_INVALID_ARG, "ttt_timing_read: NULL context");
  return fail(ctx, ctx->timing_read(kc, total_ms, launches, flops));
}
