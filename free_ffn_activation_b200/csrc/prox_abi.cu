// Host side of the libprox C ABI (see include/prox.h): argument validation,
// device checks, launch plans, workspace layout and kernel orchestration.
// Nothing here computes any step of the method; every step runs in the
// kernels of k_stage1.cu, k_stage2.cu and k_quantize.cu.
#include "prox_internal.cuh"

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#define PROX_API extern "C" __attribute__((visibility("default")))

namespace prox {

size_t stage1_smem_bytes(int d_model, int B, int NB, int unit_cap);
size_t stage2_smem_bytes(int d_model, int B, int nstage, int C, int max_ch);
int stage2_nchd(int d_model, int B);

int max_tokens_per_pass(int d_model) {
    if (d_model <= 4096) return 8;
    if (d_model <= 8192) return 4;
    return 0;
}

static int pow2_ceil(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

int tokens_per_pass(int d_model, int batch) {
    const int mx = max_tokens_per_pass(d_model);
    if (mx == 0) return 0;
    int b = batch < 1 ? 1 : batch;
    if (b > mx) b = mx;
    return pow2_ceil(b);
}

// Starting point of the Stage-1 launch plan: one CTA per SM; a CTA covers one
// or two adjacent column blocks (whichever fills more SMs), and the row
// groups of its columns form one thread-block cluster (<= 8, portable). The
// launch shrinks the cluster if not every cluster could be resident at once.
Stage1Plan stage1_plan(int d, int f, int B, int num_sms) {
    Stage1Plan p;
    p.C = f / kCB;
    int best = -1;
    for (int nb = 1; nb <= 2; ++nb) {
        if (p.C % nb) continue;
        const int groups = p.C / nb;
        int n_r = num_sms / groups;
        if (n_r < 1) n_r = 1;
        if (n_r > kS1MaxRowGroups) n_r = kS1MaxRowGroups;
        const int ctas = groups * n_r;
        if (ctas >= best) {  // on a tie, fewer and larger clusters
            best = ctas;
            p.nb_blocks = nb;
            p.n_r = n_r;
        }
    }
    // enough row groups that one CTA's rows fit in shared memory
    while (p.n_r < kS1MaxRowGroups &&
           stage1_smem_bytes(d, B, p.nb_blocks, (d + p.n_r - 1) / p.n_r) > (size_t)kS2SmemBudget)
        ++p.n_r;
    p.unit_cap = (d + p.n_r - 1) / p.n_r;
    p.depth_sel = 0;  // the launch picks the deepest ring that fits
    p.smem = stage1_smem_bytes(d, B, p.nb_blocks, p.unit_cap);
    return p;
}

Stage2Plan stage2_plan(int d, int B, int C, int max_ch) {
    Stage2Plan p;
    p.nchunk = stage2_nchd(d, B);
    // The deepest ring within the 227 KB of dynamic shared memory an sm_100
    // CTA may opt into, of at most 16 slots and 192 KB of rows (a ninth 24 KB
    // slot on the 4096-wide layer measured slower)
    constexpr size_t kSmemMax = 227 * 1024, kRingMax = 192 * 1024;
    const size_t stage = (size_t)6 * d;
    int ns = 16;
    while (ns > 0 && ((size_t)ns * stage > kRingMax ||
                      stage2_smem_bytes(d, B, ns, C, max_ch) > kSmemMax))
        --ns;
    p.nstage = ns;
    p.smem = stage2_smem_bytes(d, B, ns, C, max_ch);
    return p;
}

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

WsLayout ws_layout(int d, int f, int B) {
    (void)d;
    const size_t C = (size_t)f / kCB;
    WsLayout L;
    size_t o = 0;
    L.status = o;
    o += 256;
    L.ucount = o;
    o = align_up(o + C * 4, 256);
    L.tcount = o;
    o = align_up(o + C * B * 4, 256);
    L.ulist = o;
    o = align_up(o + C * kCB * 4, 256);
    L.tlist = o;
    o = align_up(o + (size_t)B * f * 4, 256);
    L.ug = L.tile_cnt = L.sb = L.pos_ch = o;
    L.clear_bytes = 0;
    if (B >= 4) {  // tensor-core Stage 2 (see k_stage2_umma.cu)
        L.ug = o;
        o += (size_t)f * 2 * B * 4;
        L.tile_cnt = o;
        o = align_up(o + (size_t)(f / 64) * 4, 256);
        L.clear_bytes = o - L.ug;
        L.sb = o;
        o = align_up(o + (size_t)(f / 64) * 2048, 256);
        L.pos_ch = o;
        o = align_up(o + (size_t)f * 4, 256);
    }
    L.acc = L.blk_cnt = o;
    if (B <= 4) {  // tensor-core Stage 1 (see k_stage1_tc.cu)
        L.acc = o;
        o = align_up(o + (size_t)2 * B * f * 8, 256);
        L.blk_cnt = o;
        o = align_up(o + C * 4, 256);
    }
    L.total = o;
    return L;
}

// ---------------------------------------------------------------------------
// device checks
// ---------------------------------------------------------------------------
struct DevInfo {
    int checked = 0;
    int ok = 0;
    int sms = 0;
};
static DevInfo g_dev[64];
static std::mutex g_dev_mu;

static prox_status current_device(int *sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PROX_ECUDA;
    if (dev < 0 || dev >= 64) return PROX_EDEVICE;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo &di = g_dev[dev];
    if (!di.checked) {
        int major = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return PROX_ECUDA;
        di.ok = (major == 10);
        di.sms = n;
        di.checked = 1;
    }
    if (!di.ok) return PROX_EDEVICE;
    *sms = di.sms;
    return PROX_OK;
}

cudaError_t set_max_dynamic_smem(const void *kern, size_t smem) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static std::map<std::pair<int, const void *>, size_t> done;
    std::lock_guard<std::mutex> lk(mu);
    size_t &cur = done[{dev, kern}];
    if (smem <= cur) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) cur = smem;
    return e;
}

// NULL counts as aligned: optional outputs are checked only when given
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool shape_ok(int d, int f) {
    return d >= 256 && f >= 256 && d % 256 == 0 && f % 256 == 0 && max_tokens_per_pass(d) > 0 &&
           f <= 1024 * kCB;  // Stage-2 shared memory holds per-block scans of <= 1024 blocks
}

static prox_status check_layer(const prox_layer *L, bool need_exact) {
    if (!L || !shape_ok(L->d_model, L->d_ff)) return PROX_EINVAL;
    if (L->activation != PROX_ACT_SWIGLU && L->activation != PROX_ACT_GEGLU) return PROX_EINVAL;
    if (L->proxy_kind != PROX_PROXY_INT4 && L->proxy_kind != PROX_PROXY_BF16) return PROX_EINVAL;
    if (!L->q_up || !L->q_gate || !aligned16(L->q_up) || !aligned16(L->q_gate)) return PROX_EINVAL;
    if (L->proxy_kind == PROX_PROXY_INT4 &&
        (!L->s_up || !L->s_gate || !aligned16(L->s_up) || !aligned16(L->s_gate)))
        return PROX_EINVAL;
    if (need_exact) {
        if (!L->w_up_cm || !L->w_gate_cm || !L->w_down) return PROX_EINVAL;
        if (!aligned16(L->w_up_cm) || !aligned16(L->w_gate_cm) || !aligned16(L->w_down))
            return PROX_EINVAL;
    }
    return PROX_OK;
}

static bool tau_ok(float t) { return std::isfinite(t) && t >= 0.f; }

// test hooks (set by prox_debug_set through the binding's test helpers only)
static uint32_t g_spin_limit = kDefaultWaitUs;
static int g_debug_skip = -1;
// prox_test_set_skip: which kernel's arrival CTA 0 skips (kSkip*) and where
static int g_skip_where = 0, g_skip_pos = -1;
constexpr int kSkipStage1Tc = 1, kSkipStage2Tc = 3;
// measurement hook (prox_test_set_stamps): phase stamps of the next passes
static unsigned long long *g_stamps = nullptr;

// Stage-2 and Stage-1 engines (prox_set_stage2_engine, prox_set_stage1_engine)
static std::atomic<int> g_engine{PROX_ENGINE_AUTO};
static std::atomic<int> g_engine1{PROX_ENGINE_AUTO};

// Whether a Stage-1 pass of B tokens takes the tensor-core proxy products
// of k_stage1.cu (passes of 8 tokens, or of 4 on shapes the tensor-core
// Stage 1 of k_stage1_tc.cu does not take; INT4 proxy; automatic there)
static bool use_tc1(int B, int proxy_kind) {
    return g_engine1.load() != PROX_ENGINE_SIMT && B >= 4 && proxy_kind == PROX_PROXY_INT4;
}

// Whether a Stage-1 pass of B tokens runs k_stage1_tc (passes of <= 4
// tokens, INT4 proxy, d_model <= 4096, when the tensor-core Stage-1 engine
// is selected) and its plan. The automatic choice keeps the CUDA-core
// kernel there: it streams the gathered proxy rows faster (each thread's
// copies progress on their own; a tensor-core K step waits for all of its
// 512 pieces).
static bool use_tc1_small(int d, int f, int B, int proxy_kind, int sms, int *n_r, int *cap,
                          size_t *smem) {
    if (g_engine1.load() != PROX_ENGINE_TC || proxy_kind != PROX_PROXY_INT4 || B > 4)
        return false;
    return stage1_tc_plan(d, f, B, sms, n_r, cap, smem);
}

// Whether a pass of B tokens runs the tensor-core Stage 2 (and its plan)
static bool use_tc(int d, int f, int B, int sms, Stage2UPlan *p) {
    const int e = g_engine.load();
    if (e == PROX_ENGINE_SIMT || B < 4) return false;
    // automatic: passes of 8 tokens, or of 4 on layers of d_model >= 8192
    // (whose passes hold at most 4 tokens); measured faster there
    if (e == PROX_ENGINE_AUTO && B < kTcMinBatch && !(B >= 4 && d >= 8192)) return false;
    return stage2u_plan(d, f, sms, p);
}

// One pass (nb <= tokens_per_pass tokens) of Stage 1: masks, kept-channel
// lists in the workspace, s~ when s_out is given, and y cleared when given.
static prox_status pass_stage1(const prox_layer *L, const uint16_t *x, int nb, float tau_x,
                               float tau_s, float *y_clear, uint8_t *mask_x, uint8_t *mask_s,
                               float *s_out, unsigned char *w, int sms, bool lists,
                               const float *y_init, cudaStream_t st) {
    const int d = L->d_model, f = L->d_ff;
    const int B = pow2_ceil(nb);
    const WsLayout W = ws_layout(d, f, B);
    const Stage1Plan p1 = stage1_plan(d, f, B, sms);
    Stage1Args a{};
    a.d = d;
    a.f = f;
    a.nb = nb;
    a.C = p1.C;
    a.n_r = p1.n_r;
    a.unit_cap = p1.unit_cap;
    a.x = x;
    a.tau_x = tau_x;
    a.tau_s = tau_s;
    a.q_up = L->q_up;
    a.q_gate = L->q_gate;
    a.s_up = L->s_up;
    a.s_gate = L->s_gate;
    a.y_zero = y_clear;
    a.y_init = y_clear ? y_init : nullptr;
    a.mask_x = mask_x;
    a.mask_s = mask_s;
    a.s_out = s_out;
    a.build_lists = lists ? 1 : 0;
    a.act = L->activation;
    a.pk = L->proxy_kind;
    a.tc = use_tc1(B, L->proxy_kind) ? 1 : 0;
    Stage2UPlan pu;
    if (lists && use_tc(d, f, B, sms, &pu)) {
        a.z_clear = reinterpret_cast<uint4 *>(w + W.ug);
        a.z_n16 = (int)(W.clear_bytes / 16);
    }
    a.wait_us = g_spin_limit;
    a.stamps = g_stamps;
    a.debug_skip = g_skip_where == kSkipStage1Tc ? g_skip_pos : -1;
    a.status = reinterpret_cast<uint32_t *>(w + W.status);
    a.ucount = reinterpret_cast<int32_t *>(w + W.ucount);
    a.tcount = reinterpret_cast<int32_t *>(w + W.tcount);
    a.ulist = reinterpret_cast<uint32_t *>(w + W.ulist);
    a.tlist = reinterpret_cast<int32_t *>(w + W.tlist);
    int nr = 0, cap = 0;
    size_t smem = 0;
    if (use_tc1_small(d, f, B, L->proxy_kind, sms, &nr, &cap, &smem)) {
        a.n_r = nr;
        a.unit_cap = cap;
        a.tc = 1;
        a.acc = reinterpret_cast<long long *>(w + W.acc);
        a.blk_cnt = reinterpret_cast<int32_t *>(w + W.blk_cnt);
        // the sums and block counters start from zero (the region also holds
        // other data when the workspace served another shape or batch)
        if (cudaMemsetAsync(w + W.acc, 0, W.total - W.acc, st) != cudaSuccess) return PROX_ECUDA;
        return launch_stage1_tc(B, a, smem, st) == cudaSuccess ? PROX_OK : PROX_ECUDA;
    }
    return launch_stage1(B, a, p1, st) == cudaSuccess ? PROX_OK : PROX_ECUDA;
}

// One pass of Stage 2, consuming the lists the preceding Stage 1 left in w.
static prox_status pass_stage2(const prox_layer *L, const uint16_t *x, int nb, float *y,
                               int32_t *idx_s, int32_t *count_s, unsigned char *w, int sms,
                               cudaStream_t st) {
    const int d = L->d_model, f = L->d_ff;
    const int B = pow2_ceil(nb);
    const WsLayout W = ws_layout(d, f, B);
    const int C = f / kCB;
    Stage2UPlan pu;
    if (use_tc(d, f, B, sms, &pu)) {
        Stage2UArgs u{};
        u.d = d;
        u.f = f;
        u.nb = nb;
        u.C = C;
        u.x = x;
        u.w_up = L->w_up_cm;
        u.w_gate = L->w_gate_cm;
        u.w_down = L->w_down;
        u.y = y;
        u.idx_s = idx_s;
        u.count_s = count_s;
        u.act = L->activation;
        u.ucount = reinterpret_cast<int32_t *>(w + W.ucount);
        u.tcount = reinterpret_cast<int32_t *>(w + W.tcount);
        u.ulist = reinterpret_cast<uint32_t *>(w + W.ulist);
        u.tlist = reinterpret_cast<int32_t *>(w + W.tlist);
        u.status = reinterpret_cast<uint32_t *>(w + W.status);
        u.wait_us = g_spin_limit;
        u.span = pu.span;
        u.nstage = pu.nstage;
        u.cw = pu.cw;
        u.rows_dn = pu.rows_dn;
        u.nstage_dn = pu.nstage_dn;
        u.ug = reinterpret_cast<float *>(w + W.ug);
        u.tile_cnt = reinterpret_cast<int32_t *>(w + W.tile_cnt);
        u.sb = reinterpret_cast<uint16_t *>(w + W.sb);
        u.pos_ch = reinterpret_cast<uint32_t *>(w + W.pos_ch);
        u.stamps = g_stamps;
        u.debug_skip = g_skip_where == kSkipStage2Tc ? g_skip_pos : -1;
        return launch_stage2_umma(B, u, sms, st) == cudaSuccess ? PROX_OK : PROX_ECUDA;
    }
    const int max_ch = (f + sms - 1) / sms + 1;
    const Stage2Plan p2 = stage2_plan(d, B, C, max_ch);
    if (p2.nstage < 2) return PROX_EINVAL;
    Stage2Args b{};
    b.d = d;
    b.f = f;
    b.nb = nb;
    b.C = C;
    b.x = x;
    b.w_up = L->w_up_cm;
    b.w_gate = L->w_gate_cm;
    b.w_down = L->w_down;
    b.y = y;
    b.idx_s = idx_s;
    b.act = L->activation;
    b.count_s = count_s;
    b.ucount = reinterpret_cast<int32_t *>(w + W.ucount);
    b.tcount = reinterpret_cast<int32_t *>(w + W.tcount);
    b.ulist = reinterpret_cast<uint32_t *>(w + W.ulist);
    b.tlist = reinterpret_cast<int32_t *>(w + W.tlist);
    b.status = reinterpret_cast<uint32_t *>(w + W.status);
    b.spin_limit = g_spin_limit;
    b.debug_skip = g_debug_skip;
    b.nstage = p2.nstage;
    b.max_ch = max_ch;
    b.stamps = g_stamps;
    return launch_stage2(B, p2.nchunk, b, sms, p2.smem, st) == cudaSuccess ? PROX_OK : PROX_ECUDA;
}

// Stage 1 [+ Stage 2] over `batch` tokens, in passes of at most B tokens
static prox_status run_forward(const prox_layer *L, const uint16_t *x, int batch, float tau_x,
                               float tau_s, float *y, uint8_t *mask_x, uint8_t *mask_s,
                               int32_t *idx_s, int32_t *count_s, float *s_out, void *ws,
                               size_t ws_bytes, cudaStream_t st, bool stage2,
                               const float *y_init = nullptr) {
    int sms = 0;
    prox_status ps = current_device(&sms);
    if (ps != PROX_OK) return ps;
    const int d = L->d_model, f = L->d_ff;
    const int Bmax = tokens_per_pass(d, batch);
    if (ws_bytes < ws_layout(d, f, Bmax).total) return PROX_ENOMEM;
    unsigned char *w = static_cast<unsigned char *>(ws);
    for (int t0 = 0; t0 < batch; t0 += Bmax) {
        const int nb = (batch - t0) < Bmax ? (batch - t0) : Bmax;
        const uint16_t *xt = x + (size_t)t0 * d;
        ps = pass_stage1(L, xt, nb, tau_x, tau_s, stage2 ? y + (size_t)t0 * d : nullptr,
                         mask_x ? mask_x + (size_t)t0 * d : nullptr,
                         mask_s ? mask_s + (size_t)t0 * f : nullptr,
                         s_out ? s_out + (size_t)t0 * f : nullptr, w, sms, stage2,
                         y_init ? y_init + (size_t)t0 * d : nullptr, st);
        if (ps != PROX_OK || !stage2) {
            if (ps != PROX_OK) return ps;
            continue;
        }
        ps = pass_stage2(L, xt, nb, y + (size_t)t0 * d, idx_s ? idx_s + (size_t)t0 * f : nullptr,
                         count_s ? count_s + t0 : nullptr, w, sms, st);
        if (ps != PROX_OK) return ps;
    }
    return PROX_OK;
}

}  // namespace prox

using namespace prox;

PROX_API prox_status prox_quantize_proxy(int d_model, int d_ff, const uint16_t *w_cm,
                                         uint8_t *q_out, float *scale_out, void *stream) {
    if (!w_cm || !q_out || !scale_out || !shape_ok(d_model, d_ff)) return PROX_EINVAL;
    if (!aligned16(w_cm) || !aligned16(q_out) || !aligned16(scale_out)) return PROX_EINVAL;
    int sms = 0;
    prox_status ps = current_device(&sms);
    if (ps != PROX_OK) return ps;
    if (launch_quantize(d_model, d_ff, w_cm, q_out, scale_out, (cudaStream_t)stream) !=
        cudaSuccess)
        return PROX_ECUDA;
    return PROX_OK;
}

PROX_API prox_status prox_bf16_proxy(int d_model, int d_ff, const uint16_t *w_cm,
                                     uint16_t *q16_out, void *stream) {
    if (!w_cm || !q16_out || !shape_ok(d_model, d_ff)) return PROX_EINVAL;
    if (!aligned16(w_cm) || !aligned16(q16_out)) return PROX_EINVAL;
    int sms = 0;
    prox_status ps = current_device(&sms);
    if (ps != PROX_OK) return ps;
    return launch_tile_bf16(d_model, d_ff, w_cm, q16_out, (cudaStream_t)stream) == cudaSuccess
               ? PROX_OK
               : PROX_ECUDA;
}

PROX_API size_t prox_workspace_bytes(int d_model, int d_ff, int batch) {
    if (!shape_ok(d_model, d_ff) || batch < 0) return 0;
    return ws_layout(d_model, d_ff, tokens_per_pass(d_model, batch)).total;
}

PROX_API prox_status prox_ffn_forward(const prox_layer *layer, const uint16_t *x, int batch,
                                      float tau_x, float tau_s, float *y, uint8_t *mask_x,
                                      uint8_t *mask_s, int32_t *idx_s, int32_t *count_s,
                                      void *ws, size_t ws_bytes, void *stream) {
    prox_status ps = check_layer(layer, true);
    if (ps != PROX_OK) return ps;
    if (batch < 0 || !tau_ok(tau_x) || !tau_ok(tau_s)) return PROX_EINVAL;
    if (batch == 0) return PROX_OK;
    if (!x || !y || !ws || !aligned16(x) || !aligned16(y) || !aligned16(ws)) return PROX_EINVAL;
    if (!aligned16(mask_x) || !aligned16(mask_s) || !aligned16(idx_s) || !aligned16(count_s))
        return PROX_EINVAL;
    return run_forward(layer, x, batch, tau_x, tau_s, y, mask_x, mask_s, idx_s, count_s, nullptr,
                       ws, ws_bytes, (cudaStream_t)stream, true);
}

// Allocation-free forward: the workspace is one file-scope device array per
// device, looked up once per device (see prox_ffn_forward_static in prox.h).
namespace prox {
constexpr size_t kStaticWsBytes = PROX_STATIC_WORKSPACE_BYTES;
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];
static void *g_static_ptr[64];
static std::mutex g_static_mu;

static prox_status static_workspace(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PROX_ECUDA;
    if (dev < 0 || dev >= 64) return PROX_EDEVICE;
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (!g_static_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) return PROX_ECUDA;
        g_static_ptr[dev] = p;
    }
    *out = g_static_ptr[dev];
    return PROX_OK;
}
}  // namespace prox

PROX_API prox_status prox_ffn_forward_static(const prox_layer *layer, const uint16_t *x,
                                             int batch, float tau_x, float tau_s, float *y,
                                             uint8_t *mask_x, uint8_t *mask_s, int32_t *idx_s,
                                             int32_t *count_s, void *stream) {
    prox_status ps = check_layer(layer, true);
    if (ps != PROX_OK) return ps;
    if (batch < 0 || !tau_ok(tau_x) || !tau_ok(tau_s)) return PROX_EINVAL;
    if (batch == 0) return PROX_OK;
    if (!x || !y || !aligned16(x) || !aligned16(y)) return PROX_EINVAL;
    if (!aligned16(mask_x) || !aligned16(mask_s) || !aligned16(idx_s) || !aligned16(count_s))
        return PROX_EINVAL;
    const int d = layer->d_model, f = layer->d_ff;
    if (ws_layout(d, f, tokens_per_pass(d, batch)).total > kStaticWsBytes) return PROX_ENOMEM;
    int sms = 0;
    ps = current_device(&sms);
    if (ps != PROX_OK) return ps;
    void *ws = nullptr;
    ps = static_workspace(&ws);
    if (ps != PROX_OK) return ps;
    return run_forward(layer, x, batch, tau_x, tau_s, y, mask_x, mask_s, idx_s, count_s, nullptr,
                       ws, kStaticWsBytes, (cudaStream_t)stream, true);
}

PROX_API prox_status prox_static_last_device_status(void *stream, uint32_t *flags_out) {
    void *ws = nullptr;
    prox_status ps = static_workspace(&ws);
    if (ps != PROX_OK) return ps;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemsetAsync(ws, 0, sizeof v, st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
        return PROX_ECUDA;
    if (flags_out) *flags_out = v;
    return v ? PROX_ETIMEOUT : PROX_OK;
}

static bool eps_ok(float e) { return std::isfinite(e) && e >= 0.f; }

PROX_API prox_status prox_rmsnorm_bf16(int d_model, int batch, const float *h, float eps,
                                       uint16_t *x_out, void *stream) {
    if (d_model < 256 || d_model % 256 != 0 || batch < 0 || !eps_ok(eps)) return PROX_EINVAL;
    if (batch == 0) return PROX_OK;
    if (!h || !x_out || !aligned16(h) || !aligned16(x_out)) return PROX_EINVAL;
    int sms = 0;
    prox_status ps = current_device(&sms);
    if (ps != PROX_OK) return ps;
    return launch_rmsnorm(d_model, batch, h, eps, x_out, (cudaStream_t)stream) == cudaSuccess
               ? PROX_OK
               : PROX_ECUDA;
}

PROX_API prox_status prox_ffn_block(const prox_layer *layer, const float *h_in, int batch,
                                    float tau_x, float tau_s, float eps, float *h_out,
                                    uint16_t *x_out, uint8_t *mask_x, uint8_t *mask_s,
                                    int32_t *idx_s, int32_t *count_s, void *ws, size_t ws_bytes,
                                    void *stream) {
    prox_status ps = check_layer(layer, true);
    if (ps != PROX_OK) return ps;
    if (batch < 0 || !tau_ok(tau_x) || !tau_ok(tau_s) || !eps_ok(eps)) return PROX_EINVAL;
    if (batch == 0) return PROX_OK;
    if (!h_in || !h_out || !x_out || !ws || !aligned16(h_in) || !aligned16(h_out) ||
        !aligned16(x_out) || !aligned16(ws))
        return PROX_EINVAL;
    if (!aligned16(mask_x) || !aligned16(mask_s) || !aligned16(idx_s) || !aligned16(count_s))
        return PROX_EINVAL;
    const int d = layer->d_model;
    if (ws_bytes < ws_layout(d, layer->d_ff, tokens_per_pass(d, batch)).total) return PROX_ENOMEM;
    int sms = 0;
    ps = current_device(&sms);
    if (ps != PROX_OK) return ps;
    cudaStream_t st = (cudaStream_t)stream;
    if (launch_rmsnorm(d, batch, h_in, eps, x_out, st) != cudaSuccess) return PROX_ECUDA;
    return run_forward(layer, x_out, batch, tau_x, tau_s, h_out, mask_x, mask_s, idx_s, count_s,
                       nullptr, ws, ws_bytes, st, true, h_in);
}

PROX_API int prox_max_batch_per_pass(int d_model) { return max_tokens_per_pass(d_model); }

PROX_API int prox_set_stage1_engine(int engine) {
    if (engine != PROX_ENGINE_AUTO && engine != PROX_ENGINE_SIMT && engine != PROX_ENGINE_TC)
        return -1;
    return g_engine1.exchange(engine);
}

PROX_API int prox_set_stage2_engine(int engine) {
    if (engine != PROX_ENGINE_AUTO && engine != PROX_ENGINE_SIMT && engine != PROX_ENGINE_TC)
        return -1;
    return g_engine.exchange(engine);
}

PROX_API prox_status prox_ffn_stage1(const prox_layer *layer, const uint16_t *x, int batch,
                                     float tau_x, float tau_s, float *y_clear, uint8_t *mask_x,
                                     uint8_t *mask_s, void *ws, size_t ws_bytes, void *stream) {
    prox_status ps = check_layer(layer, false);
    if (ps != PROX_OK) return ps;
    const int d = layer->d_model, f = layer->d_ff;
    if (batch < 0 || batch > max_tokens_per_pass(d) || !tau_ok(tau_x) || !tau_ok(tau_s))
        return PROX_EINVAL;
    if (batch == 0) return PROX_OK;
    if (!x || !ws || !aligned16(x) || !aligned16(ws) || !aligned16(y_clear) ||
        !aligned16(mask_x) || !aligned16(mask_s))
        return PROX_EINVAL;
    if (ws_bytes < ws_layout(d, f, tokens_per_pass(d, batch)).total) return PROX_ENOMEM;
    int sms = 0;
    ps = current_device(&sms);
    if (ps != PROX_OK) return ps;
    return pass_stage1(layer, x, batch, tau_x, tau_s, y_clear, mask_x, mask_s, nullptr,
                       static_cast<unsigned char *>(ws), sms, true, nullptr, (cudaStream_t)stream);
}

PROX_API prox_status prox_ffn_stage2(const prox_layer *layer, const uint16_t *x, int batch,
                                     float *y, int32_t *idx_s, int32_t *count_s, void *ws,
                                     size_t ws_bytes, void *stream) {
    prox_status ps = check_layer(layer, true);
    if (ps != PROX_OK) return ps;
    const int d = layer->d_model, f = layer->d_ff;
    if (batch < 0 || batch > max_tokens_per_pass(d)) return PROX_EINVAL;
    if (batch == 0) return PROX_OK;
    if (!x || !y || !ws || !aligned16(x) || !aligned16(y) || !aligned16(ws) ||
        !aligned16(idx_s) || !aligned16(count_s))
        return PROX_EINVAL;
    if (ws_bytes < ws_layout(d, f, tokens_per_pass(d, batch)).total) return PROX_ENOMEM;
    int sms = 0;
    ps = current_device(&sms);
    if (ps != PROX_OK) return ps;
    return pass_stage2(layer, x, batch, y, idx_s, count_s, static_cast<unsigned char *>(ws), sms,
                       (cudaStream_t)stream);
}

PROX_API prox_status prox_proxy_state(const prox_layer *layer, const uint16_t *x, int batch,
                                      float tau_x, float *s_out, uint8_t *mask_x, void *ws,
                                      size_t ws_bytes, void *stream) {
    prox_status ps = check_layer(layer, false);
    if (ps != PROX_OK) return ps;
    if (batch < 0 || !tau_ok(tau_x)) return PROX_EINVAL;
    if (batch == 0) return PROX_OK;
    if (!x || !s_out || !ws || !aligned16(x) || !aligned16(ws) || !aligned16(s_out) ||
        !aligned16(mask_x))
        return PROX_EINVAL;
    return run_forward(layer, x, batch, tau_x, 0.f, nullptr, mask_x, nullptr, nullptr, nullptr,
                       s_out, ws, ws_bytes, (cudaStream_t)stream, false);
}

// calibration workspace: [forward ws for the widest pass][s~ n_cal x d_ff fp32]
// [histogram 65536 u32][scratch 64 B][tau 2 x fp32]
struct CalLayout {
    size_t fwd, s, hist, scratch, tau, total;
};
static CalLayout cal_layout(int d, int f, int n_cal) {
    CalLayout c;
    size_t o = 0;
    c.fwd = o;
    o = align_up(o + prox_workspace_bytes(d, f, n_cal), 256);
    c.s = o;
    o = align_up(o + (size_t)n_cal * f * 4, 256);
    c.hist = o;
    o = align_up(o + 65536 * 4, 256);
    c.scratch = o;
    o += 64;
    c.tau = o;
    o += 64;
    c.total = o;
    return c;
}

PROX_API size_t prox_calibrate_workspace_bytes(int d_model, int d_ff, int n_cal) {
    if (!shape_ok(d_model, d_ff) || n_cal < 1) return 0;
    return cal_layout(d_model, d_ff, n_cal).total;
}

static long quantile_rank(long n, double keep) {
    double r = std::floor((1.0 - keep) * (double)n);
    long rank = (long)r;
    if (rank < 0) rank = 0;
    if (rank > n - 1) rank = n - 1;
    return rank;
}

PROX_API prox_status prox_calibrate(const prox_layer *layer, const uint16_t *x_cal, int n_cal,
                                    double keep_x, double keep_s, float *tau_x_out,
                                    float *tau_s_out, void *ws, size_t ws_bytes, void *stream) {
    prox_status ps = check_layer(layer, false);
    if (ps != PROX_OK) return ps;
    if (!x_cal || n_cal < 1 || !tau_x_out || !tau_s_out || !ws || !aligned16(x_cal) ||
        !aligned16(ws))
        return PROX_EINVAL;
    if (!(keep_x >= 0.0 && keep_x <= 1.0) || !(keep_s >= 0.0 && keep_s <= 1.0)) return PROX_EINVAL;
    const int d = layer->d_model, f = layer->d_ff;
    const CalLayout c = cal_layout(d, f, n_cal);
    if (ws_bytes < c.total) return PROX_ENOMEM;
    int sms = 0;
    ps = current_device(&sms);
    if (ps != PROX_OK) return ps;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned char *w = static_cast<unsigned char *>(ws);
    uint32_t *hist = reinterpret_cast<uint32_t *>(w + c.hist);
    uint32_t *scratch = reinterpret_cast<uint32_t *>(w + c.scratch);
    float *tau = reinterpret_cast<float *>(w + c.tau);
    const long nx = (long)n_cal * d;
    if (launch_select_bf16_abs(x_cal, nx, quantile_rank(nx, keep_x), hist, scratch, tau, st) !=
        cudaSuccess)
        return PROX_ECUDA;
    float tx = 0.f;
    if (cudaMemcpyAsync(&tx, tau, sizeof(float), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return PROX_ECUDA;
    float *s_all = reinterpret_cast<float *>(w + c.s);
    ps = run_forward(layer, x_cal, n_cal, tx, 0.f, nullptr, nullptr, nullptr, nullptr, nullptr,
                     s_all, w + c.fwd, c.s - c.fwd, st, false);
    if (ps != PROX_OK) return ps;
    const long ns = (long)n_cal * f;
    if (launch_select_f32_abs(s_all, ns, quantile_rank(ns, keep_s), hist, scratch, tau + 1, st) !=
        cudaSuccess)
        return PROX_ECUDA;
    float ts = 0.f;
    if (cudaMemcpyAsync(&ts, tau + 1, sizeof(float), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return PROX_ECUDA;
    *tau_x_out = tx;
    *tau_s_out = ts;
    return PROX_OK;
}

PROX_API prox_status prox_calibrate_histogram(const prox_layer *layer, const uint16_t *x_cal,
                                              int n_cal, double keep_x, double keep_s,
                                              long max_samples, int bins, float *tau_x_out,
                                              float *tau_s_out, void *ws, size_t ws_bytes,
                                              void *stream) {
    prox_status ps = check_layer(layer, false);
    if (ps != PROX_OK) return ps;
    if (!x_cal || n_cal < 1 || !tau_x_out || !tau_s_out || !ws || !aligned16(x_cal) ||
        !aligned16(ws))
        return PROX_EINVAL;
    if (!(keep_x >= 0.0 && keep_x <= 1.0) || !(keep_s >= 0.0 && keep_s <= 1.0)) return PROX_EINVAL;
    if (max_samples < 1 || bins < 1024 || bins > 65536 || bins % 1024 != 0) return PROX_EINVAL;
    const int d = layer->d_model, f = layer->d_ff;
    const CalLayout c = cal_layout(d, f, n_cal);
    if (ws_bytes < c.total) return PROX_ENOMEM;
    int sms = 0;
    ps = current_device(&sms);
    if (ps != PROX_OK) return ps;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned char *w = static_cast<unsigned char *>(ws);
    uint32_t *hist = reinterpret_cast<uint32_t *>(w + c.hist);
    uint32_t *scratch = reinterpret_cast<uint32_t *>(w + c.scratch);
    float *tau = reinterpret_cast<float *>(w + c.tau);
    // every k-th of n pooled values, k = ceil(n / max_samples); the rank counts samples
    auto stride = [&](long n) { return (n + max_samples - 1) / max_samples; };
    auto samples = [&](long n) { return (n + stride(n) - 1) / stride(n); };
    const long nx = (long)n_cal * d;
    if (launch_hist_quantile_bf16(x_cal, nx, stride(nx), quantile_rank(samples(nx), keep_x), bins,
                                  hist, scratch, tau, st) != cudaSuccess)
        return PROX_ECUDA;
    float tx = 0.f;
    if (cudaMemcpyAsync(&tx, tau, sizeof(float), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return PROX_ECUDA;
    float *s_all = reinterpret_cast<float *>(w + c.s);
    ps = run_forward(layer, x_cal, n_cal, tx, 0.f, nullptr, nullptr, nullptr, nullptr, nullptr,
                     s_all, w + c.fwd, c.s - c.fwd, st, false);
    if (ps != PROX_OK) return ps;
    const long ns = (long)n_cal * f;
    if (launch_hist_quantile_f32(s_all, ns, stride(ns), quantile_rank(samples(ns), keep_s), bins,
                                 hist, scratch, tau + 1, st) != cudaSuccess)
        return PROX_ECUDA;
    float ts = 0.f;
    if (cudaMemcpyAsync(&ts, tau + 1, sizeof(float), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return PROX_ECUDA;
    *tau_x_out = tx;
    *tau_s_out = ts;
    return PROX_OK;
}

PROX_API prox_status prox_allocate(double e, double alpha, double s1_max, double s2_anchor,
                                   double *s1_out, double *s2_out) {
    if (!s1_out || !s2_out || !(alpha > 0.0) || !(e >= 0.0 && e <= 1.0) ||
        !(s1_max >= 0.0 && s1_max <= 1.0) || !(s2_anchor >= 0.0 && s2_anchor <= 1.0))
        return PROX_EINVAL;
    double s2 = s2_anchor;
    double s1 = 1.0 - 3.0 * (s2 - e) / (2.0 * alpha);
    if (s1 > s1_max || s1 < 0.0) {
        s1 = s1 > s1_max ? s1_max : 0.0;
        s2 = e + 2.0 * alpha * (1.0 - s1) / 3.0;
    }
    *s1_out = s1;
    *s2_out = s2;
    return PROX_OK;
}

PROX_API prox_status prox_last_device_status(void *ws, size_t ws_bytes, void *stream,
                                             uint32_t *flags_out) {
    if (!ws || ws_bytes < 256) return PROX_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemsetAsync(ws, 0, sizeof v, st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
        return PROX_ECUDA;
    if (flags_out) *flags_out = v;
    return v ? PROX_ETIMEOUT : PROX_OK;
}

PROX_API const char *prox_status_str(prox_status s) {
    switch (s) {
        case PROX_OK: return "ok";
        case PROX_EINVAL: return "invalid argument";
        case PROX_ENOMEM: return "workspace too small";
        case PROX_ECUDA: return "CUDA error";
        case PROX_ETIMEOUT: return "device-side wait timed out";
        case PROX_EDEVICE: return "current device is not compute capability 10.x (B200)";
    }
    return "unknown status";
}

// Test hooks, not part of prox.h: shorten the bounded waits and make the
// Stage-2 producer of CTA 0 skip one channel position, so that a test can
// exercise the timeout path without faulting anything.
PROX_API void prox_test_set_wait(uint32_t spin_limit, int skip_position) {
    prox::g_spin_limit = spin_limit ? spin_limit : kDefaultWaitUs;
    prox::g_debug_skip = skip_position;
}

// Test hook, not part of prox.h: in CTA 0 of the tensor-core kernels, one
// arrival never happens, so that a bounded wait runs out (see prox_testing.h)
PROX_API void prox_test_set_skip(int where, int position) {
    prox::g_skip_where = where;
    prox::g_skip_pos = position;
}

// Measurement hook, not part of prox.h: passes launched while `slots` is set
// record %globaltimer phase stamps (prox::StampSlot) into it.
PROX_API void prox_test_set_stamps(unsigned long long *slots) { prox::g_stamps = slots; }
