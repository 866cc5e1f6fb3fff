// C ABI of libgdnscan.so: argument checks, workspace layout and the launch plan.
//
// The plan for one call (SANA-WM blog, blog.hotdry.top: recurrence in section
// 混合线性注意力, span composition and prologue order in the Context-Parallel
// section; reverse scan with block resets per the hyper.ai summary, 方法):
//   [prologue]  RMSNorm -> ReLU -> key scale -> RoPE on raw q, k   (a1)
//   contract    A_t, U_t for every frame-head                     (a2)
//   per direction:
//     chunked:    compose (E_p, H_p, g_p) per span                (a3)
//                 prefix over spans -> span start states          (a4)
//                 replay each span from its start state           (a5)
//     sequential: one chain over T                                (a4+a5)
//     blocks:     one chain per reset block                       (a5)
//     readout     O_t = Q_t S_t^T                                 (a6)
#include <stdio.h>
#include <string.h>

#include <cmath>
#include <string>
#include <vector>

#include "gdn_internal.cuh"

namespace gdn {

static thread_local std::string t_last_error;
static thread_local long long t_launches = 0;

void count_launch(int n) { t_launches += n; }

// ---- phase timing with CUDA events (gdn_profile_enable / gdn_profile_read) ----
enum Phase {
  PH_PROLOGUE = 0, PH_CONTRACT, PH_COMPOSE, PH_PREFIX, PH_SCAN, PH_READOUT, PH_SCAN_READOUT,
  PH_CONTRACT_SCAN, PH_BWD_RECOMPUTE, PH_BWD_W, PH_BWD_ADJOINT, PH_BWD_FRAME, PH_BWD_TOKENS,
  PH_BWD_DQ, PH_COUNT
};
struct ProfRec {
  int phase;
  cudaEvent_t a, b;
};
struct Profiler {
  bool on = false;
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> pool;
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
  void recycle() {
    for (auto& r : recs) {
      pool.push_back(r.a);
      pool.push_back(r.b);
    }
    recs.clear();
  }
};
static thread_local Profiler t_prof;

struct PhaseScope {
  cudaStream_t st;
  int idx = -1;
  PhaseScope(int phase, cudaStream_t s) : st(s) {
    if (!t_prof.on) return;
    ProfRec r{phase, t_prof.get(), t_prof.get()};
    cudaEventRecord(r.a, st);
    t_prof.recs.push_back(r);
    idx = (int)t_prof.recs.size() - 1;
  }
  ~PhaseScope() {
    if (idx >= 0) cudaEventRecord(t_prof.recs[idx].b, st);
  }
};

static int fail(int status, const char* fmt, const char* detail = "") {
  char buf[512];
  snprintf(buf, sizeof(buf), fmt, detail);
  t_last_error = buf;
  return status;
}

// Host-side fault injection (gdn_fault_inject): the next t_inject scan calls
// on this host thread report a launch failure once their arguments have been
// checked, before they allocate or launch anything.
static thread_local int t_inject = 0;

static int injected_failure() {
  if (t_inject <= 0) return GDN_OK;
  --t_inject;
  return fail(GDN_ERR_CUDA, "injected launch failure (gdn_fault_inject)%s");
}

static int cuda_fail(cudaError_t e, const char* where) {
  char buf[512];
  snprintf(buf, sizeof(buf), "%s: %s", where, cudaGetErrorString(e));
  t_last_error = buf;
  return GDN_ERR_CUDA;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static bool valid_D(int D) { return D == 16 || D == 32 || D == 64 || D == 128 || D == 256; }

static int block_len(unsigned flags) {
  int b = (int)GDN_BLOCK(flags);
  return b ? b : 3;
}
static int chunk_len(unsigned flags) {
  int c = (int)GDN_CHUNK(flags);
  return c ? c : 8;
}

Layout make_layout(int B, int H, int T, int S, int D, unsigned flags) {
  Layout L;
  const size_t heads = (size_t)B * H;
  const size_t frames = heads * T;
  const size_t mat = (size_t)D * D * sizeof(float);
  const int nchunk = (T + chunk_len(flags) - 1) / chunk_len(flags);
  const int nblock = (T + block_len(flags) - 1) / block_len(flags);
  L.nseg_max = nchunk > nblock ? nchunk : nblock;
  size_t off = 0;
  L.A = off;
  off = align256(off + frames * mat);
  L.U = off;
  off = align256(off + frames * mat);
  L.Sfr = off;
  off = align256(off + frames * mat);  // fp32, or bf16 hi+lo: the same bytes
  L.Sfr2 = L.Sfr;
  if (flags & GDN_BIDIR) {             // the reverse direction's per-frame states
    L.Sfr2 = off;
    off = align256(off + frames * mat);
  }
  L.E = off;
  off = align256(off + heads * L.nseg_max * mat);
  L.Hc = off;
  off = align256(off + heads * L.nseg_max * mat);
  L.Sst = off;
  off = align256(off + heads * L.nseg_max * mat);
  L.g = off;
  off = align256(off + heads * L.nseg_max * sizeof(float));
  L.flags = off;  // per frame-head publication counters of the overlapped plan
  off = align256(off + frames * sizeof(int));
  L.qh = L.kh = off;
  if (flags & GDN_FUSED_PROLOGUE) {
    const size_t elt = (flags & GDN_BF16) ? 2 : 4;
    const size_t tens = frames * (size_t)S * D * elt;
    L.qh = off;
    off = align256(off + tens);
    L.kh = off;
    off = align256(off + tens);
  }
  L.total = off;
  return L;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static int device_cc_major() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return 0;
  return major;
}

static int check_sizes(int B, int H, int T, int S, int D) {
  if (B < 1 || H < 1 || T < 1 || S < 1)
    return fail(GDN_ERR_INVALID, "sizes must be >= 1%s");
  if (!valid_D(D)) return fail(GDN_ERR_UNSUPPORTED, "D must be 16, 32, 64, 128 or 256%s");
  if (S > 65535 * 64) return fail(GDN_ERR_UNSUPPORTED, "S above 4194240%s");
  const long long frames = (long long)B * H * T;
  if (frames > (1LL << 31) - 1) return fail(GDN_ERR_UNSUPPORTED, "B*H*T too large%s");
  return GDN_OK;
}

// Runs one direction of the scan from A, U already in the workspace.
static int run_direction(const gdn_params& p, const Layout& L, char* ws, bool reverse,
                         bool block_reset, const void* q, void* out, float* state_out,
                         bool use_tc_chain, bool use_tc_readout, const ProArgs* pro_q,
                         cudaStream_t st, size_t sfr_off, bool do_readout) {
  const bool bf16 = (p.flags & GDN_BF16) != 0;
  const long long frames = (long long)p.B * p.H * p.T;
  ChainArgs a;
  memset(&a, 0, sizeof(a));
  a.D = p.D;
  a.T = p.T;
  a.L = chunk_len(p.flags);
  a.block = block_len(p.flags);
  a.reverse = reverse ? 1 : 0;
  a.heads = p.B * p.H;
  a.A = (const float*)(ws + L.A);
  a.U = (const float*)(ws + L.U);
  a.gamma = p.gamma;
  a.state_in = reverse && (p.flags & GDN_BIDIR) && (p.flags & GDN_REV_STATE_IN) ? p.state_in_rev
                                                                              : p.state_in;
  a.state_out = state_out;
  a.Sfr = (float*)(ws + sfr_off);
  a.sfr_hilo = use_tc_readout ? 1 : 0;
  a.E = (float*)(ws + L.E);
  a.Hc = (float*)(ws + L.Hc);
  a.g = (float*)(ws + L.g);
  a.Sst = (float*)(ws + L.Sst);
  a.y_image = use_tc_chain ? 1 : 0;  // the tensor-core chains read A and E as operand images
  a.e_image = a.y_image;
  a.sst_hilo = a.y_image;

  auto chain = [&](const ChainArgs& c, int n) -> cudaError_t {
    PhaseScope ps(c.mode == CHAIN_COMPOSE ? PH_COMPOSE : c.mode == CHAIN_PREFIX ? PH_PREFIX : PH_SCAN,
                  st);
    return use_tc_chain ? tc_chain(c, n, st) : simt_chain(c, n, st);
  };
  cudaError_t e;
  // Replay fused with the readout: spans or reset blocks, tensor-core path, no prologue.
  const bool fused = do_readout && (p.flags & GDN_FUSED_REPLAY) && use_tc_chain && use_tc_readout &&
                     !pro_q && (p.flags & GDN_BF16) &&
                     !(p.flags & GDN_SEQUENTIAL) && tc_scan_readout_supported(p.D);
  auto scan_readout = [&](const ChainArgs& c, int n) -> int {
    PhaseScope ps(PH_SCAN_READOUT, st);
    cudaError_t er = tc_scan_readout(c, n, q, out, p.S, st);
    return er == cudaSuccess ? GDN_OK : cuda_fail(er, "scan+readout");
  };
  if (fused) {
    a.mode = CHAIN_SCAN;
    if (block_reset) {
      a.seg = SEG_BLOCKS;
      a.nseg = (p.T + a.block - 1) / a.block;
      return scan_readout(a, a.heads * a.nseg);
    }
    a.seg = SEG_CHUNKS;
    a.nseg = (p.T + a.L - 1) / a.L;
    if (a.nseg > 1) {
      a.mode = CHAIN_COMPOSE;
      if ((e = chain(a, 2 * a.heads * a.nseg)) != cudaSuccess) return cuda_fail(e, "compose");
      a.mode = CHAIN_PREFIX;
      if ((e = chain(a, a.heads)) != cudaSuccess) return cuda_fail(e, "prefix");
      a.mode = CHAIN_SCAN;
    }
    return scan_readout(a, a.heads * a.nseg);
  }
  if (p.flags & GDN_SEQUENTIAL) {
    a.seg = SEG_SEQUENTIAL;
    a.seq_reset = block_reset ? 1 : 0;
    a.nseg = 1;
    a.mode = CHAIN_SCAN;
    if ((e = chain(a, a.heads)) != cudaSuccess) return cuda_fail(e, "scan chain");
  } else if (block_reset) {
    a.seg = SEG_BLOCKS;
    a.nseg = (p.T + a.block - 1) / a.block;
    a.mode = CHAIN_SCAN;
    if ((e = chain(a, a.heads * a.nseg)) != cudaSuccess) return cuda_fail(e, "block chains");
  } else {
    a.seg = SEG_CHUNKS;
    a.nseg = (p.T + a.L - 1) / a.L;
    if (a.nseg == 1) {
      a.mode = CHAIN_SCAN;
      if ((e = chain(a, a.heads)) != cudaSuccess) return cuda_fail(e, "scan chain");
    } else {
      a.mode = CHAIN_COMPOSE;
      if ((e = chain(a, 2 * a.heads * a.nseg)) != cudaSuccess) return cuda_fail(e, "compose");
      a.mode = CHAIN_PREFIX;
      if ((e = chain(a, a.heads)) != cudaSuccess) return cuda_fail(e, "prefix");
      a.mode = CHAIN_SCAN;
      if ((e = chain(a, a.heads * a.nseg)) != cudaSuccess) return cuda_fail(e, "replay");
    }
  }
  if (!do_readout) return GDN_OK;
  {
    PhaseScope ps(PH_READOUT, st);
    if (use_tc_readout)
      e = tc_readout(q, ws + sfr_off, out, frames, p.S, p.D, pro_q, st);
    else
      e = simt_readout(bf16, q, (const float*)(ws + sfr_off), out, frames, p.S, p.D, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "readout");
  return GDN_OK;
}

static int scan_ex(const gdn_params& p, cudaStream_t st) {
  int rc = check_sizes(p.B, p.H, p.T, p.S, p.D);
  if (rc) return rc;
  const unsigned f = p.flags;
  if (!p.q || !p.k || !p.v || !p.beta || !p.gamma || !p.out)
    return fail(GDN_ERR_INVALID, "null q/k/v/beta/gamma/out%s");
  if (!aligned16(p.q) || !aligned16(p.k) || !aligned16(p.v) || !aligned16(p.out) ||
      !aligned16(p.beta) || !aligned16(p.gamma))
    return fail(GDN_ERR_INVALID, "pointers must be 16-byte aligned%s");
  if (p.out == p.q || p.out == p.k || p.out == p.v)
    return fail(GDN_ERR_INVALID, "out must not alias q, k or v%s");
  if ((f & GDN_BIDIR) && (!p.out_rev || p.out_rev == p.out || !aligned16(p.out_rev)))
    return fail(GDN_ERR_INVALID, "GDN_BIDIR needs a separate, aligned out_rev%s");
  if ((f & GDN_BIDIR) && (f & GDN_REVERSE))
    return fail(GDN_ERR_INVALID, "GDN_BIDIR and GDN_REVERSE are exclusive%s");
  if ((f & GDN_SEQUENTIAL) && (f & GDN_CHUNKED))
    return fail(GDN_ERR_INVALID, "GDN_SEQUENTIAL and GDN_CHUNKED are exclusive%s");
  if ((f & GDN_UCPE) && !(f & GDN_FUSED_PROLOGUE))
    return fail(GDN_ERR_INVALID, "GDN_UCPE is part of GDN_FUSED_PROLOGUE%s");
  if ((f & GDN_UCPE) && (!p.ucpe_q || !p.ucpe_k || !aligned16(p.ucpe_q) || !aligned16(p.ucpe_k)))
    return fail(GDN_ERR_INVALID, "GDN_UCPE needs 16-byte aligned ucpe_q and ucpe_k%s");
  if (f & GDN_FUSED_PROLOGUE) {
    if (!p.w_q || !p.w_k) return fail(GDN_ERR_INVALID, "prologue needs w_q and w_k%s");
    if (p.grid_h < 1 || p.grid_w < 1 || (long long)p.grid_h * p.grid_w != p.S)
      return fail(GDN_ERR_INVALID, "prologue needs grid_h * grid_w == S%s");
    if (f & GDN_KEYS_SCALED)
      return fail(GDN_ERR_INVALID, "GDN_FUSED_PROLOGUE applies the key scale itself%s");
  }
  const Layout L = make_layout(p.B, p.H, p.T, p.S, p.D, f);
  if (!p.workspace || p.workspace_bytes < L.total)
    return fail(GDN_ERR_WORKSPACE, "workspace missing or smaller than gdn_workspace_bytes%s");
  if (((uintptr_t)p.workspace & 255u) != 0)
    return fail(GDN_ERR_INVALID, "workspace must be 256-byte aligned%s");
  if ((rc = injected_failure()) != GDN_OK) return rc;

  const bool bf16 = (f & GDN_BF16) != 0;
  const bool sm100 = device_cc_major() == 10;
  const bool simt = (f & GDN_FORCE_SIMT) || !bf16 || !sm100;
  const bool tc_contract_ok = !simt && tc_contract_supported(p.D);
  const bool tc_readout_ok = !simt && tc_readout_supported(p.D);
  // D = 256 has tensor-core chains for whole-scan chains only (sequential,
  // or one per reset block): its plan is sequential unless spans are asked for.
  const bool seq_plan = (f & GDN_SEQUENTIAL) ||
                        (p.D == 256 && !simt && !(f & (GDN_CHUNKED | GDN_FUSED_REPLAY)));
  const bool tc_chain_ok = !simt && (tc_chain_supported(p.D) || (p.D == 256 && seq_plan));
  char* ws = (char*)p.workspace;
  const long long frames = (long long)p.B * p.H * p.T;
  cudaError_t e;

  const void* q = p.q;
  const void* k = p.k;
  bool keys_scaled = (f & GDN_KEYS_SCALED) != 0;
  ProArgs pro_k = {}, pro_q = {};
  const ProArgs* ppk = nullptr;
  const ProArgs* ppq = nullptr;
  if (f & GDN_FUSED_PROLOGUE) {
    const float eps = p.eps > 0.f ? p.eps : 1e-6f;
    const float base = p.rope_base > 0.f ? p.rope_base : 10000.f;
    const int npos_max = p.grid_h > p.grid_w ? p.grid_h : p.grid_w;
    if (tc_contract_ok && tc_readout_ok && p.D == 128 && npos_max <= tc_prologue_max_positions()) {
      // Fused: the tensor-core loaders apply RMSNorm, ReLU and RoPE to the raw
      // tiles in shared memory; the key scale goes into the contraction's
      // epilogue constants (RoPE is linear, so the order does not matter).
      // Each CTA computes its (cos, sin) table into shared memory at start-up.
      const int npos = p.grid_h > p.grid_w ? p.grid_h : p.grid_w;
      const bool cam = (f & GDN_UCPE) != 0;
      pro_k = ProArgs{p.w_k, p.grid_w, eps, npos, base, cam ? p.ucpe_k : nullptr, p.H, p.T};
      pro_q = ProArgs{p.w_q, p.grid_w, eps, npos, base, cam ? p.ucpe_q : nullptr, p.H, p.T};
      ppk = &pro_k;
      ppq = &pro_q;
    } else {
      const float ks = (float)(1.0 / std::sqrt((double)p.D * (double)p.S));
      {
        PhaseScope ps(PH_PROLOGUE, st);
        e = simt_prologue(bf16, p.q, p.k, p.w_q, p.w_k, ws + L.qh, ws + L.kh, frames, p.S,
                          p.grid_w, p.D, eps, base, ks, st, (f & GDN_UCPE) ? p.ucpe_q : nullptr,
                          (f & GDN_UCPE) ? p.ucpe_k : nullptr, p.H, p.T);
      }
      if (e != cudaSuccess) return cuda_fail(e, "prologue");
      q = ws + L.qh;
      k = ws + L.kh;
      keys_scaled = true;
    }
  }
  const double c = keys_scaled ? 1.0 : 1.0 / std::sqrt((double)p.D * (double)p.S);
  float* A = (float*)(ws + L.A);
  float* U = (float*)(ws + L.U);
  const bool block_reset = (f & GDN_BLOCK_RESET) != 0;

  // Sequential chains alongside the contraction (one cooperative launch),
  // then the readout: the plan unless chunks or separate launches are asked
  // for, or the shape does not fit it.
  const bool bidir = (f & GDN_BIDIR) != 0;
  const int ndir = bidir ? 2 : 1;
  // Very few frame-heads (at most a quarter of the SMs): cut each frame-head's
  // tokens over several CTAs (partial sums), then the chains in their own
  // launch. From a quarter on, the chains alongside the contraction win (one
  // 3-frame block of 16 heads, 48 frame-heads at 720p: 0.149 against 0.168 ms
  // per call).
  const int nsms = (tc_contract_ok && p.D == 128) ? tc_num_sms() : 0;
  const int nst = (p.S + 63) / 64;
  const bool split = tc_contract_ok && tc_chain_ok && tc_readout_ok && p.D == 128 &&
                     !(f & GDN_FUSED_REPLAY) && frames * 4 <= nsms && nst >= 4;
  int parts = 1;
  if (split) {  // 2 <= parts <= nst / 2: every part holds at least 2 stages
    parts = (int)(nsms / frames);
    if (parts > nst / 2) parts = nst / 2;
    if (parts > 8) parts = 8;
  }
  const bool overlap = !split && tc_contract_ok && tc_chain_ok && tc_readout_ok &&
                       tc_overlap_supported(p.D) && !(f & (GDN_CHUNKED | GDN_NO_OVERLAP |
                                                          GDN_FUSED_REPLAY)) &&
                       (!bidir || (block_reset && tc_readout2_supported(p.D))) &&
                       ndir * p.B * p.H <= tc_overlap_max_chains();
  if (overlap) {
    OvlArgs o;
    memset(&o, 0, sizeof(o));
    o.heads = p.B * p.H;
    o.T = p.T;
    o.block = block_len(f);
    o.ndir = ndir;
    o.gamma = p.gamma;
    o.A = (const uint8_t*)A;
    o.flags = (int*)(ws + L.flags);
    if (bidir) {
      // forward never reset; reverse reset per block, run block by block
      o.dir[0] = OvlDir{0, 0, 0, p.state_in, p.state_out, 0};
      o.dir[1] = OvlDir{1, 1, 0, (f & GDN_REV_STATE_IN) ? p.state_in_rev : p.state_in,
                        p.state_out_rev, 0};
    } else {
      o.dir[0] = OvlDir{(f & GDN_REVERSE) ? 1 : 0, 0, block_reset ? 1 : 0, p.state_in,
                        p.state_out, 0};
    }
    o.a_image = 1;
    o.contract_rev = o.dir[0].reverse && !o.dir[0].blocks_asc;
    // one chain per head reads each frame's A_t image and U_t once: their L2
    // lines are dropped after that read instead of being written back (the
    // A_t images stay for a later gdn_frame_scan_bwd when asked to)
    if (!bidir) o.discard = 1 | ((f & GDN_SAVE_FOR_BACKWARD) ? 0 : 2);
    {
      PhaseScope ps(PH_CONTRACT_SCAN, st);
      e = tc_contract_scan(k, p.v, p.beta, A, U, frames, p.S, (float)(c * c), (float)c, ppk, o,
                           ws + L.Sfr, bidir ? ws + L.Sfr2 : nullptr, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "contract + sequential scan");
    PhaseScope ps(PH_READOUT, st);
    if (bidir)
      e = tc_readout2(q, ws + L.Sfr, ws + L.Sfr2, p.out, p.out_rev, frames, p.S, p.D, ppq, st);
    else
      e = tc_readout(q, ws + L.Sfr, p.out, frames, p.S, p.D, ppq, st);
    if (e != cudaSuccess) return cuda_fail(e, "readout");
    return GDN_OK;
  }
  {
    PhaseScope ps(PH_CONTRACT, st);
    if (split) {
      float* Aacc = (float*)(ws + L.Sfr);  // free until the chains store the states
      e = tc_contract_split(k, p.v, p.beta, Aacc, U, frames, p.S, (float)(c * c), (float)c, parts,
                            ppk, st);
      if (e == cudaSuccess) e = tc_to_image(Aacc, A, frames, p.D, st);
    } else if (tc_contract_ok)
      e = tc_contract(k, p.v, p.beta, A, U, frames, p.S, p.D, (float)(c * c), (float)c,
                      tc_chain_ok ? 1 : 0, ppk, st);
    else
      e = simt_contract(bf16, k, p.v, p.beta, A, U, frames, p.S, p.D, (float)(c * c), (float)c,
                        st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "contract");

  gdn_params pp = p;
  if (seq_plan) pp.flags |= GDN_SEQUENTIAL;
  if (f & GDN_BIDIR) {
    // Both directions' states first, then (tensor-core path) one readout that
    // reads each Q tile once for both outputs.
    const bool both = tc_readout_ok && tc_chain_ok && tc_readout2_supported(p.D);
    rc = run_direction(pp, L, ws, false, false, q, p.out, p.state_out, tc_chain_ok,
                       tc_readout_ok, ppq, st, L.Sfr, !both);
    if (rc) return rc;
    rc = run_direction(pp, L, ws, true, block_reset, q, p.out_rev, p.state_out_rev, tc_chain_ok,
                       tc_readout_ok, ppq, st, L.Sfr2, !both);
    if (rc || !both) return rc;
    PhaseScope ps(PH_READOUT, st);
    e = tc_readout2(q, ws + L.Sfr, ws + L.Sfr2, p.out, p.out_rev, frames, p.S, p.D, ppq, st);
    if (e != cudaSuccess) return cuda_fail(e, "bidirectional readout");
    return GDN_OK;
  }
  return run_direction(pp, L, ws, (f & GDN_REVERSE) != 0, block_reset, q, p.out, p.state_out,
                       tc_chain_ok, tc_readout_ok, ppq, st, L.Sfr, true);
}

// ---- backward --------------------------------------------------------------
// The tensor-core backward (D = 128, bf16) keeps per-frame matrices only; the
// CUDA-core one also stages three fp32 token products.
static bool bwd_tc_by_flags(int D, unsigned flags) {
  return D == 128 && (flags & GDN_BF16) && !(flags & GDN_FORCE_SIMT);
}

struct BwdLayout {
  size_t A, U, Sfr, W, G, dM, Bimg, zero, flags, s0, P2, P3, P5, total;
};

static BwdLayout make_bwd_layout(int B, int H, int T, int S, int D, unsigned f) {
  BwdLayout L;
  const size_t frames = (size_t)B * H * T;
  const size_t mat = frames * D * D * sizeof(float);
  const size_t tok = frames * S * D * sizeof(float);
  const bool tc = bwd_tc_by_flags(D, f);
  size_t off = 0;
  size_t* mats[] = {&L.A, &L.U, &L.Sfr, &L.W, &L.G, &L.dM};
  for (size_t* m : mats) {
    *m = off;
    off = align256(off + mat);
  }
  L.Bimg = L.zero = L.flags = L.s0 = L.P2 = L.P3 = L.P5 = off;
  if (tc) {
    L.s0 = off;  // state_in as bf16 hi/lo pairs
    off = align256(off + (size_t)B * H * 2 * D * D * 2);
    L.Bimg = off;  // per frame [dA + dA^T ; G] bf16, 64 KiB
    off = align256(off + frames * 65536);
    L.zero = off;  // an all-zero operand image
    off = align256(off + (size_t)kImageBytes);
    L.flags = off;  // publication counters of the overlapped recompute
    off = align256(off + frames * sizeof(int));
  } else {
    size_t* toks[] = {&L.P2, &L.P3, &L.P5};
    for (size_t* m : toks) {
      *m = off;
      off = align256(off + tok);
    }
  }
  L.total = off;
  return L;
}

// Tensor-core backward, D = 128, bf16: recompute with the forward kernels
// (states as bf16 hi/lo pairs), W = dO^T Q by the contraction, G by the
// adjoint chain, per-frame terms, token gradients and dq on tensor cores.
static int scan_bwd_tc(const gdn_bwd_params& p, char* ws, size_t oA, size_t oU, size_t oSfr,
                       size_t oW, size_t oG, size_t oS0, size_t oB, size_t oZero, size_t oFlags,
                       cudaStream_t st) {
  const unsigned f = p.flags;
  const bool reverse = (f & GDN_REVERSE) != 0;
  const bool block_reset = (f & GDN_BLOCK_RESET) != 0;
  const int block = block_len(f);
  const long long frames = (long long)p.B * p.H * p.T;
  const int heads = p.B * p.H;
  const double c = (f & GDN_KEYS_SCALED) ? 1.0 : 1.0 / std::sqrt((double)p.D * (double)p.S);
  float* A = (float*)(ws + oA);
  float* U = (float*)(ws + oU);
  float* W = (float*)(ws + oW);
  cudaError_t e;
  const bool saved = p.saved_workspace != nullptr;
  if (saved) {
    // the forward call's A_t images and states (their offsets do not depend on flags)
    const Layout Lf = make_layout(p.B, p.H, p.T, p.S, p.D, GDN_BF16);
    A = (float*)((char*)p.saved_workspace + Lf.A);
  }
  // 1. recompute A_t (operand images), U_t and the states S_t (hi/lo pairs)
  ChainArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = CHAIN_SCAN;
  a.seg = SEG_SEQUENTIAL;
  a.D = 128;
  a.T = p.T;
  a.L = 1;
  a.block = block;
  a.seq_reset = block_reset ? 1 : 0;
  a.reverse = reverse ? 1 : 0;
  a.nseg = 1;
  a.heads = heads;
  a.A = A;
  a.U = U;
  a.gamma = p.gamma;
  a.state_in = p.state_in;
  a.Sfr = saved ? (float*)((char*)p.saved_workspace + make_layout(p.B, p.H, p.T, p.S, p.D, GDN_BF16).Sfr)
                : (float*)(ws + oSfr);
  a.sfr_hilo = 1;
  a.y_image = 1;
  if (!saved) {
    PhaseScope ps(PH_BWD_RECOMPUTE, st);
    if (heads <= tc_overlap_max_chains()) {
      OvlArgs o;
      memset(&o, 0, sizeof(o));
      o.heads = heads;
      o.T = p.T;
      o.block = block;
      o.ndir = 1;
      o.gamma = p.gamma;
      o.A = (const uint8_t*)A;
      o.flags = (int*)(ws + oFlags);
      o.dir[0] = OvlDir{a.reverse, 0, a.seq_reset, p.state_in, nullptr, 0};
      o.a_image = 1;
      o.contract_rev = a.reverse;
      e = tc_contract_scan(p.k, p.v, p.beta, A, U, frames, p.S, (float)(c * c), (float)c, nullptr,
                           o, a.Sfr, nullptr, st);
    } else {
      e = tc_contract(p.k, p.v, p.beta, A, U, frames, p.S, 128, (float)(c * c), (float)c, 1,
                      nullptr, st);
      if (e == cudaSuccess) e = tc_chain(a, heads, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "backward: recompute");
  }
  // 2./3. W_t = dO_t^T Q_t (the contraction's U with keys := q, values := dO,
  // beta = 1) and the adjoint chain for G_t (hi/lo pairs): side by side in one
  // launch when the chains fit, the contraction visiting frames in the
  // adjoint's order; else one after the other
  ChainArgs b = a;
  b.mode = CHAIN_ADJOINT;
  b.Zw = W;
  b.Gout = (float*)(ws + oG);
  b.dS_out = p.d_state_out;
  b.zero_img = ws + oZero;
  e = cudaMemsetAsync(ws + oZero, 0, kImageBytes, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward: zero image");
  if (heads <= tc_overlap_max_chains()) {
    PhaseScope ps(PH_BWD_ADJOINT, st);
    OvlArgs w;
    memset(&w, 0, sizeof(w));
    w.heads = heads;
    w.T = p.T;
    w.block = block;
    w.ndir = 1;
    w.gamma = p.gamma;
    w.A = (const uint8_t*)A;
    w.flags = (int*)(ws + oFlags);
    w.zero_img = (const uint8_t*)(ws + oZero);
    w.a_image = 2;  // keep the recomputed A_t images
    w.contract_rev = !a.reverse;
    w.dir[0] = OvlDir{a.reverse, 0, a.seq_reset, p.d_state_out, nullptr, 1};
    e = tc_contract_scan(p.q, p.d_out, nullptr, A, W, frames, p.S, 1.f, 1.f, nullptr, w, b.Gout,
                         nullptr, st);
    if (e != cudaSuccess) return cuda_fail(e, "backward: dO^T Q + adjoint chain");
  } else {
    {
      PhaseScope ps(PH_BWD_W, st);
      e = tc_contract(p.q, p.d_out, nullptr, A, W, frames, p.S, 128, 1.f, 1.f, 2, nullptr, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "backward: dO^T Q");
    PhaseScope ps(PH_BWD_ADJOINT, st);
    e = tc_chain(b, heads, st);
    if (e != cudaSuccess) return cuda_fail(e, "backward: adjoint chain");
  }
  // 4. per frame: dM = S'^T G, dA + dA^T and dgamma, the token kernel's operand
  {
    PhaseScope ps(PH_BWD_FRAME, st);
    e = tc_bwd_frames(a.Sfr, p.state_in, ws + oS0, ws + oZero, b.Gout, A, p.gamma, p.dgamma,
                      ws + oB, frames, heads, p.T, a.reverse, a.seq_reset, block, st);
    if (e == cudaSuccess && p.d_state_in)
      e = simt_bwd_ds0(b.Gout, A, p.gamma, p.d_state_in, heads, p.T, frame_at(0, p.T, a.reverse),
                       st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "backward: per-frame terms");
  // 5. token gradients and dq
  {
    PhaseScope ps(PH_BWD_TOKENS, st);
    e = tc_bwd_tokens(p.k, p.v, p.beta, ws + oB, p.dk, p.dv, p.dbeta, frames, p.S, (float)c, st);
  }
  if (e == cudaSuccess) {
    PhaseScope ps(PH_BWD_DQ, st);
    e = tc_readout_trans(p.d_out, a.Sfr, p.dq, frames, p.S, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "backward: token gradients");
  return GDN_OK;
}

static int scan_bwd(const gdn_bwd_params& p, cudaStream_t st) {
  int rc = check_sizes(p.B, p.H, p.T, p.S, p.D);
  if (rc) return rc;
  const unsigned f = p.flags;
  const unsigned allowed = GDN_BF16 | GDN_REVERSE | GDN_BLOCK_RESET | GDN_KEYS_SCALED |
                           GDN_FORCE_SIMT | (0xffu << 8) | (0xffu << 16);
  if (f & ~allowed) return fail(GDN_ERR_INVALID, "gdn_frame_scan_bwd: unsupported flag%s");
  if (!p.q || !p.k || !p.v || !p.beta || !p.gamma || !p.d_out || !p.dq || !p.dk || !p.dv ||
      !p.dbeta || !p.dgamma)
    return fail(GDN_ERR_INVALID, "null input or gradient pointer%s");
  const void* ptrs[] = {p.q, p.k, p.v, p.beta, p.gamma, p.d_out, p.dq, p.dk, p.dv, p.dbeta,
                        p.dgamma};
  for (const void* x : ptrs)
    if (!aligned16(x)) return fail(GDN_ERR_INVALID, "pointers must be 16-byte aligned%s");
  const void* outs[] = {p.dq, p.dk, p.dv};
  const void* ins[] = {p.q, p.k, p.v, p.d_out};
  for (const void* o : outs)
    for (const void* i : ins)
      if (o == i) return fail(GDN_ERR_INVALID, "gradients must not alias inputs%s");
  const BwdLayout L = make_bwd_layout(p.B, p.H, p.T, p.S, p.D, f);
  if (!p.workspace || p.workspace_bytes < L.total)
    return fail(GDN_ERR_WORKSPACE, "workspace missing or smaller than gdn_bwd_workspace_bytes%s");
  if (((uintptr_t)p.workspace & 255u) != 0)
    return fail(GDN_ERR_INVALID, "workspace must be 256-byte aligned%s");
  if ((rc = injected_failure()) != GDN_OK) return rc;

  const bool bf16 = (f & GDN_BF16) != 0;
  const bool reverse = (f & GDN_REVERSE) != 0;
  const bool block_reset = (f & GDN_BLOCK_RESET) != 0;
  const int block = block_len(f);
  const long long frames = (long long)p.B * p.H * p.T;
  const double c = (f & GDN_KEYS_SCALED) ? 1.0 : 1.0 / std::sqrt((double)p.D * (double)p.S);
  char* ws = (char*)p.workspace;
  float* A = (float*)(ws + L.A);
  float* U = (float*)(ws + L.U);
  float* Sfr = (float*)(ws + L.Sfr);
  float* W = (float*)(ws + L.W);
  float* G = (float*)(ws + L.G);
  float* dM = (float*)(ws + L.dM);
  float* P2 = (float*)(ws + L.P2);
  float* P3 = (float*)(ws + L.P3);
  float* P5 = (float*)(ws + L.P5);
  cudaError_t e;
  if (p.saved_workspace && !bwd_tc_by_flags(p.D, f))
    return fail(GDN_ERR_INVALID, "saved_workspace needs the tensor-core backward (bf16, D = 128)%s");
  if (bwd_tc_by_flags(p.D, f)) {
    if (device_cc_major() != 10)
      return fail(GDN_ERR_UNSUPPORTED, "bf16 D = 128 backward runs on sm_100 (else pass GDN_FORCE_SIMT)%s");
    return scan_bwd_tc(p, ws, L.A, L.U, L.Sfr, L.W, L.G, L.s0, L.Bimg, L.zero, L.flags, st);
  }
  // 1. forward recompute: A_t, U_t, then the states S_t (one chain per head)
  e = simt_contract(bf16, p.k, p.v, p.beta, A, U, frames, p.S, p.D, (float)(c * c), (float)c, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward: contract");
  ChainArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = CHAIN_SCAN;
  a.seg = SEG_SEQUENTIAL;
  a.D = p.D;
  a.T = p.T;
  a.L = 1;
  a.block = block;
  a.seq_reset = block_reset ? 1 : 0;
  a.reverse = reverse ? 1 : 0;
  a.nseg = 1;
  a.heads = p.B * p.H;
  a.A = A;
  a.U = U;
  a.gamma = p.gamma;
  a.state_in = p.state_in;
  a.Sfr = Sfr;
  if ((e = simt_chain(a, a.heads, st)) != cudaSuccess) return cuda_fail(e, "backward: states");
  // 2. W_t = dO_t^T Q_t (the contraction's U with keys := q, values := dO, beta = 1)
  e = simt_contract(bf16, p.q, p.d_out, nullptr, nullptr, W, frames, p.S, p.D, 1.f, 1.f, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward: dO^T Q");
  // 3. adjoint chain: G_t per frame, and the state_in gradient
  ChainArgs b = a;
  b.mode = CHAIN_ADJOINT;
  b.Zw = W;
  b.Gout = G;
  b.dS_out = p.d_state_out;
  b.dS_in = p.d_state_in;
  if ((e = simt_chain(b, b.heads, st)) != cudaSuccess) return cuda_fail(e, "backward: adjoint chain");
  // 4. per frame: dM = S'^T G -> dA + dA^T, dgamma
  e = simt_bwd_dm(Sfr, p.state_in, G, dM, frames, p.T, p.D, a.reverse, a.seq_reset, block, false,
                  st);
  if (e == cudaSuccess)
    e = simt_bwd_dterm(dM, A, false, p.gamma, p.dgamma, frames, p.D, nullptr, nullptr, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward: per-frame terms");
  // 5. per token: K^ (dA + dA^T), V G, K^ G^T, dQ = dO S_t; then dk, dv, dbeta
  e = simt_rowmat(bf16, true, 0, p.k, dM, P2, frames, p.S, p.D, (float)c, st);
  if (e == cudaSuccess) e = simt_rowmat(bf16, true, 1, p.v, G, P3, frames, p.S, p.D, 1.f, st);
  if (e == cudaSuccess) e = simt_rowmat(bf16, true, 0, p.k, G, P5, frames, p.S, p.D, (float)c, st);
  if (e == cudaSuccess) e = simt_rowmat(bf16, !bf16, 1, p.d_out, Sfr, p.dq, frames, p.S, p.D, 1.f, st);
  if (e == cudaSuccess)
    e = simt_bwd_combine(bf16, p.k, p.beta, P2, P3, P5, p.dk, p.dv, p.dbeta, frames * p.S, p.D,
                         (float)c, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward: token gradients");
  return GDN_OK;
}

int scan_ex_entry(const gdn_params& p, cudaStream_t st) {
  t_last_error.clear();
  return scan_ex(p, st);
}

int set_last_error(int status, const char* msg) {
  t_last_error = msg;
  return status;
}

}  // namespace gdn

using namespace gdn;

extern "C" {

int gdn_version(void) { return 100; }

const char* gdn_status_string(int s) {
  switch (s) {
    case GDN_OK: return "ok";
    case GDN_ERR_INVALID: return "invalid argument";
    case GDN_ERR_UNSUPPORTED: return "unsupported size";
    case GDN_ERR_CUDA: return "CUDA error";
    case GDN_ERR_TIMEOUT: return "device wait timed out";
    case GDN_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

const char* gdn_last_error(void) { return t_last_error.c_str(); }

int gdn_fault_inject(int n) {
  const int pending = t_inject;
  t_inject = n > 0 ? n : 0;
  return pending;
}

long long gdn_launch_count(int reset) {
  long long n = t_launches;
  if (reset) t_launches = 0;
  return n;
}

int gdn_frame_scan_bwd(const gdn_bwd_params* p, gdn_stream_t stream) {
  t_last_error.clear();
  if (!p) return fail(GDN_ERR_INVALID, "null params%s");
  return scan_bwd(*p, (cudaStream_t)stream);
}

size_t gdn_bwd_workspace_bytes(int B, int H, int T, int S, int D, unsigned flags) {
  (void)flags;
  if (B < 1 || H < 1 || T < 1 || S < 1 || D < 1) return 0;
  return make_bwd_layout(B, H, T, S, D, flags).total;
}

size_t gdn_workspace_bytes(int B, int H, int T, int S, int D, unsigned flags) {
  if (B < 1 || H < 1 || T < 1 || S < 1 || !valid_D(D)) return 0;
  return make_layout(B, H, T, S, D, flags).total;
}

int gdn_frame_scan_fwd_ex(const gdn_params* p, gdn_stream_t stream) {
  t_last_error.clear();
  if (!p) return fail(GDN_ERR_INVALID, "null params%s");
  return scan_ex(*p, (cudaStream_t)stream);
}

int gdn_frame_scan_fwd(const void* q, const void* k, const void* v, const float* beta,
                       const float* gamma, const float* state_in, void* out, float* state_out,
                       int B, int H, int T, int S, int D, unsigned flags, gdn_stream_t stream) {
  t_last_error.clear();
  if (flags & (GDN_FUSED_PROLOGUE | GDN_BIDIR))
    return fail(GDN_ERR_INVALID, "GDN_FUSED_PROLOGUE / GDN_BIDIR need gdn_frame_scan_fwd_ex%s");
  int rc = check_sizes(B, H, T, S, D);
  if (rc) return rc;
  gdn_params p;
  memset(&p, 0, sizeof(p));
  p.q = q;
  p.k = k;
  p.v = v;
  p.beta = beta;
  p.gamma = gamma;
  p.state_in = state_in;
  p.out = out;
  p.state_out = state_out;
  p.B = B;
  p.H = H;
  p.T = T;
  p.S = S;
  p.D = D;
  p.flags = flags;
  p.workspace_bytes = make_layout(B, H, T, S, D, flags).total;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMallocAsync(&p.workspace, p.workspace_bytes, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
  rc = scan_ex(p, st);
  e = cudaFreeAsync(p.workspace, st);
  if (rc == GDN_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(workspace)");
  return rc;
}

static int qk_prologue(const void* q_raw, const void* k_raw, const float* w_q, const float* w_k,
                       const float* ucpe_q, const float* ucpe_k, void* q_out, void* k_out, int B,
                       int H, int T, int grid_h, int grid_w, int D, float eps, float rope_base,
                       unsigned flags, cudaStream_t stream) {
  if (grid_h < 1 || grid_w < 1) return fail(GDN_ERR_INVALID, "grid must be >= 1%s");
  const long long S = (long long)grid_h * grid_w;
  if (S > 65535 * 64) return fail(GDN_ERR_UNSUPPORTED, "S above 4194240%s");
  int rc = check_sizes(B, H, T, (int)S, D);
  if (rc) return rc;
  if (!q_raw || !k_raw || !w_q || !w_k || !q_out || !k_out)
    return fail(GDN_ERR_INVALID, "null pointer%s");
  if (q_out == q_raw || q_out == k_raw || k_out == q_raw || k_out == k_raw || q_out == k_out)
    return fail(GDN_ERR_INVALID, "outputs must not alias inputs%s");
  const float ks = (float)(1.0 / std::sqrt((double)D * (double)S));
  cudaError_t e = simt_prologue((flags & GDN_BF16) != 0, q_raw, k_raw, w_q, w_k, q_out, k_out,
                                (long long)B * H * T, (int)S, grid_w, D,
                                eps > 0.f ? eps : 1e-6f, rope_base > 0.f ? rope_base : 10000.f,
                                ks, stream, ucpe_q, ucpe_k, H, T);
  if (e != cudaSuccess) return cuda_fail(e, "prologue");
  return GDN_OK;
}

int gdn_qk_prologue(const void* q_raw, const void* k_raw, const float* w_q, const float* w_k,
                    void* q_out, void* k_out, int B, int H, int T, int grid_h, int grid_w, int D,
                    float eps, float rope_base, unsigned flags, gdn_stream_t stream) {
  t_last_error.clear();
  return qk_prologue(q_raw, k_raw, w_q, w_k, nullptr, nullptr, q_out, k_out, B, H, T, grid_h,
                     grid_w, D, eps, rope_base, flags, (cudaStream_t)stream);
}

int gdn_qk_prologue_ucpe(const void* q_raw, const void* k_raw, const float* w_q, const float* w_k,
                         const float* ucpe_q, const float* ucpe_k, void* q_out, void* k_out,
                         int B, int H, int T, int grid_h, int grid_w, int D, float eps,
                         float rope_base, unsigned flags, gdn_stream_t stream) {
  t_last_error.clear();
  if (!ucpe_q || !ucpe_k || !aligned16(ucpe_q) || !aligned16(ucpe_k))
    return fail(GDN_ERR_INVALID, "ucpe_q and ucpe_k must be 16-byte aligned device pointers%s");
  return qk_prologue(q_raw, k_raw, w_q, w_k, ucpe_q, ucpe_k, q_out, k_out, B, H, T, grid_h,
                     grid_w, D, eps, rope_base, flags, (cudaStream_t)stream);
}

int gdn_frame_contract(const void* k, const void* v, const float* beta, float* A, float* U,
                       int N, int S, int D, unsigned flags, gdn_stream_t stream) {
  t_last_error.clear();
  int rc = check_sizes(1, 1, N, S, D);
  if (rc) return rc;
  if (!k || !v || !beta || !A || !U) return fail(GDN_ERR_INVALID, "null pointer%s");
  const bool bf16 = (flags & GDN_BF16) != 0;
  const double c = (flags & GDN_KEYS_SCALED) ? 1.0 : 1.0 / std::sqrt((double)D * (double)S);
  const bool tc = bf16 && !(flags & GDN_FORCE_SIMT) && device_cc_major() == 10 &&
                  tc_contract_supported(D);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = tc ? tc_contract(k, v, beta, A, U, N, S, D, (float)(c * c), (float)c, 0,
                                   nullptr, st)
                     : simt_contract(bf16, k, v, beta, A, U, N, S, D, (float)(c * c),
                                     (float)c, st);
  if (e != cudaSuccess) return cuda_fail(e, "contract");
  return GDN_OK;
}

int gdn_cp_shard_composite(const void* k, const void* v, const float* beta, const float* gamma,
                           float* E, float* H, float* g, int B, int Hh, int T, int S, int D,
                           unsigned flags, void* workspace, size_t workspace_bytes,
                           gdn_stream_t stream) {
  t_last_error.clear();
  int rc = check_sizes(B, Hh, T, S, D);
  if (rc) return rc;
  if (!k || !v || !beta || !gamma || !E || !H || !g)
    return fail(GDN_ERR_INVALID, "null pointer%s");
  if (flags & ~(GDN_BF16 | GDN_KEYS_SCALED | GDN_FORCE_SIMT | (0xffu << 8) | (0xffu << 16)))
    return fail(GDN_ERR_INVALID, "gdn_cp_shard_composite: unsupported flag%s");
  const Layout L = make_layout(B, Hh, T, S, D, flags);
  if (!workspace || workspace_bytes < L.total)
    return fail(GDN_ERR_WORKSPACE, "workspace missing or smaller than gdn_workspace_bytes%s");
  if (((uintptr_t)workspace & 255u) != 0)
    return fail(GDN_ERR_INVALID, "workspace must be 256-byte aligned%s");
  cudaStream_t st = (cudaStream_t)stream;
  const bool bf16 = (flags & GDN_BF16) != 0;
  const bool simt = (flags & GDN_FORCE_SIMT) || !bf16 || device_cc_major() != 10;
  const bool tc_chain_ok = !simt && tc_chain_supported(D);  // composes on tensor cores
  const bool tc_contract_ok = !simt && tc_contract_supported(D);
  const long long frames = (long long)B * Hh * T;
  const double c = (flags & GDN_KEYS_SCALED) ? 1.0 : 1.0 / std::sqrt((double)D * (double)S);
  char* ws = (char*)workspace;
  float* A = (float*)(ws + L.A);
  float* U = (float*)(ws + L.U);
  cudaError_t e;
  if (tc_contract_ok)
    e = tc_contract(k, v, beta, A, U, frames, S, D, (float)(c * c), (float)c, tc_chain_ok ? 1 : 0,
                    nullptr, st);
  else
    e = simt_contract(bf16, k, v, beta, A, U, frames, S, D, (float)(c * c), (float)c, st);
  if (e != cudaSuccess) return cuda_fail(e, "shard composite: contract");
  ChainArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = CHAIN_COMPOSE;
  a.seg = SEG_CHUNKS;
  a.D = D;
  a.T = T;
  a.L = T;  // one span: the whole shard
  a.block = 3;
  a.nseg = 1;
  a.heads = B * Hh;
  a.A = A;
  a.U = U;
  a.gamma = gamma;
  a.E = E;
  a.Hc = H;
  a.g = g;
  a.y_image = tc_chain_ok ? 1 : 0;
  a.e_image = 0;  // E in fp32 for the exchange
  e = tc_chain_ok ? tc_chain(a, 2 * a.heads, st) : simt_chain(a, 2 * a.heads, st);
  if (e != cudaSuccess) return cuda_fail(e, "shard composite: compose");
  return GDN_OK;
}

int gdn_cp_prefix(const float* E_all, const float* H_all, const float* g_all,
                  const float* state_in, float* S_start, int R, int r, int heads, int D,
                  gdn_stream_t stream) {
  t_last_error.clear();
  if (R < 1 || r < 0 || r >= R || heads < 1) return fail(GDN_ERR_INVALID, "bad rank or sizes%s");
  if (!valid_D(D)) return fail(GDN_ERR_UNSUPPORTED, "D must be 16, 32, 64, 128 or 256%s");
  if (!E_all || !H_all || !g_all || !S_start) return fail(GDN_ERR_INVALID, "null pointer%s");
  cudaError_t e = simt_cp_prefix(E_all, H_all, g_all, state_in, S_start, r, heads, D,
                                 (cudaStream_t)stream);
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, "cp prefix");
}

int gdn_chunk_composites(const float* A, const float* U, const float* gamma, float* E, float* Hc,
                         float* g, int N, int L, int D, unsigned flags, gdn_stream_t stream) {
  t_last_error.clear();
  int rc = check_sizes(1, N, L, 1, D);
  if (rc) return rc;
  if (!A || !U || !gamma || !E || !Hc || !g) return fail(GDN_ERR_INVALID, "null pointer%s");
  ChainArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = CHAIN_COMPOSE;
  a.seg = SEG_CHUNKS;
  a.D = D;
  a.T = L;
  a.L = L;
  a.block = 3;
  a.nseg = 1;
  a.heads = N;
  a.A = A;
  a.U = U;
  a.gamma = gamma;
  a.E = E;
  a.Hc = Hc;
  a.g = g;
  const bool tc = !(flags & GDN_FORCE_SIMT) && device_cc_major() == 10 && tc_chain_supported(D);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (tc) {
    // The tensor-core chains read A as operand images: convert into scratch.
    void* img = nullptr;
    e = cudaMallocAsync(&img, (size_t)N * L * D * D * 4, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(images)");
    e = tc_to_image(A, img, (long long)N * L, D, st);
    if (e == cudaSuccess) {
      a.A = (const float*)img;
      a.y_image = 1;
      a.e_image = 0;
      e = tc_chain(a, 2 * N, st);
    }
    cudaError_t e2 = cudaFreeAsync(img, st);
    if (e == cudaSuccess) e = e2;
  } else {
    e = simt_chain(a, 2 * N, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "compose");
  return GDN_OK;
}

int gdn_profile_enable(int enable) {
  if (enable) t_prof.recycle();
  t_prof.on = enable != 0;
  return GDN_OK;
}

int gdn_profile_read(double* ms, long long* counts, int n) {
  if (!ms || !counts || n < 1) return fail(GDN_ERR_INVALID, "null or empty output%s");
  const int np = n < PH_COUNT ? n : PH_COUNT;
  for (int i = 0; i < np; ++i) {
    ms[i] = 0.0;
    counts[i] = 0;
  }
  for (auto& r : t_prof.recs) {
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e != cudaSuccess) return cuda_fail(e, "profile event");
    float t = 0.f;
    e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(e, "profile elapsed");
    if (r.phase < np) {
      ms[r.phase] += t;
      counts[r.phase] += 1;
    }
  }
  return np;
}

int gdn_selftest_wait(int arrive, long long limit_ns, gdn_stream_t stream) {
  t_last_error.clear();
  if (limit_ns < 0 || limit_ns > 1000000000LL)
    return fail(GDN_ERR_INVALID, "limit_ns must be in [0, 1e9]%s");
  cudaError_t e = tc_selftest_wait(arrive, limit_ns, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return GDN_OK;
}

int gdn_rope_eval(int npos, int D, float rope_base, int reduced, float* cs, gdn_stream_t stream) {
  t_last_error.clear();
  if (!cs || !aligned16(cs)) return fail(GDN_ERR_INVALID, "cs must be a 16-byte aligned device pointer%s");
  if (npos < 1 || npos > (1 << 20) || !valid_D(D) || !(rope_base > 1.0f))
    return fail(GDN_ERR_INVALID, "need 1 <= npos <= 2^20, a supported D and rope_base > 1%s");
  const float base = rope_base;
  cudaError_t e = reduced ? rope_reduced((float2*)cs, npos, D, base, (cudaStream_t)stream)
                          : rope_table((float2*)cs, npos, D, base, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "rope eval launch");
  return GDN_OK;
}

int gdn_check_device_status(gdn_stream_t stream) {
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int status = 0;
  e = tc_read_status(&status, st);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (status) {
    char code[32];
    snprintf(code, sizeof(code), "%d", status);
    return fail(GDN_ERR_TIMEOUT, "a device-side wait ran out (wait code %s)", code);
  }
  return GDN_OK;
}

}  // extern "C"
