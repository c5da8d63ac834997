// Internal declarations of libprox: launch plans, workspace layout, kernel
// argument blocks and the inline-PTX helpers (mbarriers with bounded waits,
// bulk copies, vector reductions) the sm_100a kernels share.
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "prox.h"

namespace prox {

// ---------------------------------------------------------------------------
// Fixed tiling constants
// ---------------------------------------------------------------------------
constexpr int kCB = 256;            // channels per Stage-1 column block
constexpr int kS1Threads = 512;     // Stage-1 CTA size (one CTA per SM)
constexpr int kS1MaxRowGroups = 8;  // row groups per block = cluster size (portable <= 8)
constexpr int kMaxB = 8;            // tokens per pass (per-token masks)
constexpr int kS2SmemBudget = 224 * 1024;   // opt-in dynamic smem per CTA

// status word bits (first word of the workspace)
constexpr uint32_t kStTimeoutFull = 1u << 0;   // consumer waited for a stage
constexpr uint32_t kStTimeoutEmpty = 1u << 1;  // producer waited for a free slot
constexpr uint32_t kStTimeoutRed = 1u << 2;    // consumers waited for partials
constexpr uint32_t kStTimeoutDrain = 1u << 3;  // producer waited for its copies
constexpr uint32_t kStTimeoutRing = 1u << 4;   // Stage 1 waited for a ring slot
constexpr uint32_t kStTimeoutMma = 1u << 5;    // tensor-core Stage 2 waited for its MMAs

// smallest pass (tokens) the automatic engine choice sends to the
// tensor-core Stage 2 (4 on layers of d_model >= 8192)
constexpr int kTcMinBatch = 8;

// default wall-clock bound of a device-side wait, in microseconds
constexpr uint32_t kDefaultWaitUs = 2000000u;

// Phase stamps (measurement hook prox_test_set_stamps): %globaltimer values
// of one forward pass, each the minimum or maximum over the kernel's CTAs
enum StampSlot : int {
    kS1Entry = 0,    // min: a Stage-1 CTA starts
    kS1Go = 1,       // min: past griddepcontrol.wait (the previous kernel is done)
    kS1GoMax = 2,    // max: the same
    kS1Pro = 3,      // max: masks, ranks and scaled x ready (stream starts)
    kS1Stream = 4,   // max: the CTA's proxy products are done
    kS1Red = 5,      // max: the cluster's partials are summed (CTA 0)
    kS1End = 6,      // max: a Stage-1 CTA is done (lists written)
    kS2Entry = 8,    // min: a Stage-2 CTA starts
    kS2Go = 9,       // min: past griddepcontrol.wait (Stage 1 is done)
    kS2GoMax = 10,   // max: the same
    kS2List = 11,    // max: the CTA's channel list is ready
    kS2First = 12,   // min: first ring stage full
    kS2FirstMax = 13,  // max: the same
    kS2Stream = 14,  // max: the last channel of a CTA is accumulated
    kS2End = 15,     // max: a CTA's y reductions are issued
    kStampSlots = 16
};

// ---------------------------------------------------------------------------
// Host-side plans
// ---------------------------------------------------------------------------
struct Stage1Plan {
    int C;          // column blocks = d_ff / kCB
    int nb_blocks;  // column blocks per CTA (1 or 2)
    int n_r;        // row groups = cluster size; grid = C / nb_blocks * n_r
    int unit_cap;   // max units (kept rows) one CTA may own
    int depth_sel;  // Stage-1 copy ring depth: deepest >> depth_sel rows per thread
    size_t smem;    // dynamic shared memory bytes
};

struct Stage2Plan {
    int nchunk;     // 16-byte chunks of a d_model row per Stage-2 down thread
    int nstage;     // stages in the bulk-copy ring
    size_t smem;    // dynamic shared memory bytes
};

// tokens per pass for a given d_model (register budget of Stage 2 and smem of
// Stage 1); 0 if d_model is beyond what the kernels support
int max_tokens_per_pass(int d_model);
int tokens_per_pass(int d_model, int batch);   // 1, 2, 4 or 8
Stage1Plan stage1_plan(int d_model, int d_ff, int B, int num_sms);
Stage2Plan stage2_plan(int d_model, int B, int C, int max_ch);

// Launch plan of the tensor-core (union GEMM) Stage 2
struct Stage2UPlan {
    int span;       // union tiles one up/gate CTA may touch
    int nstage;     // up/gate ring stages
    int cw;         // output coordinates per down stage (512 or 256)
    int rows_dn;    // union positions one down CTA may touch
    int nstage_dn;  // down ring stages
};
bool stage2u_plan(int d_model, int d_ff, int num_sms, Stage2UPlan *p);

// Workspace layout of one forward pass (B tokens). Offsets in bytes. The
// tensor-core Stage 2 (B >= 4) adds fp32 partial sums of u and g per union
// position with the split counters right after them (one region Stage 1
// clears), the s tiles and the channel of every union position.
struct WsLayout {
    size_t status, ucount, tcount, ulist, tlist, ug, tile_cnt, sb, pos_ch, acc, blk_cnt, total;
    size_t clear_bytes;  // ug .. tile_cnt end
};
WsLayout ws_layout(int d_model, int d_ff, int B);

// ---------------------------------------------------------------------------
// Kernel argument blocks
// ---------------------------------------------------------------------------
struct Stage1Args {
    int d, f, nb;                // nb active tokens of this pass (<= B)
    int C, n_r, unit_cap, depth_sel;
    const uint16_t *x;           // [nb][d]
    float tau_x, tau_s;
    const uint8_t *q_up, *q_gate;
    const float *s_up, *s_gate;
    float *y_zero;               // [nb][d] zeroed here (Stage 2 accumulates), or null
    const float *y_init;         // [nb][d] copied into y_zero instead of zeros, or null
    uint8_t *mask_x;             // [nb][d] or null
    uint8_t *mask_s;             // [nb][f] or null
    float *s_out;                // [nb][f] or null
    int build_lists;             // write ulist/tlist/counts for Stage 2
    int act;                     // gate activation (PROX_ACT_*)
    int pk;                      // proxy kind (PROX_PROXY_*): q_up/q_gate INT4 or bf16 tiles
    int tc;                      // tensor-core proxy products (B 4 or 8, INT4 proxy)
    uint4 *z_clear;              // region cleared for the tensor-core Stage 2, or null
    int z_n16;                   // its size in 16-byte words
    uint32_t wait_us;            // wall-clock bound of each wait, microseconds
    unsigned long long *stamps;  // phase stamps (StampSlot) or null
    int debug_skip;              // test hook: in CTA 0 of a tensor-core pass, this K
                                 // step (group) never completes (-1: off)
    // workspace
    uint32_t *status;
    long long *acc;              // tensor-core Stage 1 (<= 4 tokens): [2][B][f] exact
                                 // int64 proxy sums, cleared before the pass
    int32_t *blk_cnt;            // [C] CTAs done per column block, cleared before the pass
    int32_t *ucount;             // [C]
    int32_t *tcount;             // [C][B]
    uint32_t *ulist;             // [C][kCB]  channel | token bits << 24
    int32_t *tlist;              // [B][f]
};

struct Stage2Args {
    int d, f, nb, C;
    const uint16_t *x;           // [nb][d]
    const uint16_t *w_up, *w_gate, *w_down;
    float *y;                    // [nb][d], zeroed by Stage 1
    int32_t *idx_s;              // [nb][f] or null
    int32_t *count_s;            // [nb] or null
    int act;                     // gate activation (PROX_ACT_*)
    const int32_t *ucount, *tcount;
    const uint32_t *ulist;
    const int32_t *tlist;
    uint32_t *status;
    uint32_t spin_limit;         // wall-clock bound of each wait, microseconds
    int debug_skip;              // test hook: producer never fills this
                                 // channel position of CTA 0 (-1: off)
    int nstage;
    int max_ch;                  // capacity of the per-CTA channel list
    unsigned long long *stamps;  // phase stamps (StampSlot) or null
};

struct Stage2UArgs {
    int d, f, nb, C;
    const uint16_t *x;           // [nb][d]
    const uint16_t *w_up, *w_gate, *w_down;
    float *y;                    // [nb][d], cleared (or seeded) by Stage 1
    int32_t *idx_s;              // [nb][f] or null
    int32_t *count_s;            // [nb] or null
    int act;                     // gate activation (PROX_ACT_*)
    const int32_t *ucount, *tcount;
    const uint32_t *ulist;
    const int32_t *tlist;
    uint32_t *status;
    uint32_t wait_us;            // wall-clock bound of each wait, microseconds
    int span, nstage;            // up/gate plan
    int cw, rows_dn, nstage_dn;  // down plan
    float *ug;                   // [f][2][B] partial u, g per union position (cleared)
    int32_t *tile_cnt;           // [f / 64] K blocks summed per tile (cleared)
    uint16_t *sb;                // [f / 64][2][8][64] s hi / lo tiles, 128-byte swizzled
    uint32_t *pos_ch;            // [f] union entry per position
    unsigned long long *stamps;  // phase stamps (StampSlot: entry, go, end) or null
    int debug_skip;              // test hook: the up/gate loaders of CTA 0 never
                                 // complete this step (-1: off)
};

cudaError_t launch_stage2_umma(int B, const Stage2UArgs &a, int grid, cudaStream_t s);

cudaError_t launch_stage1(int B, const Stage1Args &a, const Stage1Plan &p,
                          cudaStream_t s);
// tensor-core Stage 1 for passes of <= 4 tokens (k_stage1_tc.cu): its plan
// (false if the shape is outside it) and launch (grid a.C * a.n_r)
bool stage1_tc_plan(int d_model, int d_ff, int B, int num_sms, int *n_r, int *unit_cap,
                    size_t *smem);
cudaError_t launch_stage1_tc(int B, const Stage1Args &a, size_t smem, cudaStream_t s);
cudaError_t launch_stage2(int B, int nchunk, const Stage2Args &a, int grid,
                          size_t smem, cudaStream_t s);
cudaError_t launch_rmsnorm(int d, int nb, const float *h, float eps, uint16_t *x,
                           cudaStream_t s);
// histogram threshold of |v| over every k-th of n values (see k_quantize.cu)
cudaError_t launch_hist_quantile_bf16(const uint16_t *v, long n, long k, long rank, int bins,
                                      uint32_t *hist, uint32_t *scratch, float *tau_dev,
                                      cudaStream_t s);
cudaError_t launch_hist_quantile_f32(const float *v, long n, long k, long rank, int bins,
                                     uint32_t *hist, uint32_t *scratch, float *tau_dev,
                                     cudaStream_t s);
cudaError_t launch_quantize(int d, int f, const uint16_t *w_cm, uint8_t *q,
                            float *scale, cudaStream_t s);
// bf16 proxy: block-tiled copy [f/256][d][256] of a channel-major [f][d] weight
cudaError_t launch_tile_bf16(int d, int f, const uint16_t *w_cm, uint16_t *q16, cudaStream_t s);
// exact order statistic of |values| (bf16 or fp32 bit patterns) on device;
// writes the selected magnitude's fp32 value to *tau_dev
cudaError_t launch_select_bf16_abs(const uint16_t *v, long n, long rank,
                                   uint32_t *hist, uint32_t *scratch,
                                   float *tau_dev, cudaStream_t s);
cudaError_t launch_select_f32_abs(const float *v, long n, long rank,
                                  uint32_t *hist, uint32_t *scratch,
                                  float *tau_dev, cudaStream_t s);

// Raise a kernel's dynamic shared-memory limit to at least `smem` bytes on the
// current device (the attribute is per device; set once per device and kernel,
// thread-safe)
cudaError_t set_max_dynamic_smem(const void *kern, size_t smem);

// Launch with programmatic stream serialization (PDL): the kernel may start
// while the previous kernel in the stream finishes; it must execute
// griddepcontrol.wait before touching anything that kernel writes.
template <typename Kern, typename Args>
inline cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              const Args &args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args);
}

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
#ifdef __CUDACC__

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// try_wait with a suspend-time hint: a waiting thread sleeps until the phase
// completes (or about 0.5 ms pass) instead of spinning on the issue slots
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(500000u)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// phase stamps: no-ops unless the pass was launched with a stamp buffer
__device__ __forceinline__ void stamp_min(unsigned long long *st, int k) {
    if (st) atomicMin(st + k, (unsigned long long)global_ns());
}
__device__ __forceinline__ void stamp_max(unsigned long long *st, int k) {
    if (st) atomicMax(st + k, (unsigned long long)global_ns());
}

// Bounded wait on the phase of `bar` with the given parity: gives up and
// returns false once `limit_us` microseconds of wall time have passed.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t limit_us) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    const uint64_t lim = (uint64_t)limit_us * 1000u;
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > lim) return false;
    return true;
}

// 1-D bulk copy global -> shared, completing on an mbarrier (TMA engine).
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// L2 policy for data read once per pass (the weight streams): evicted first,
// so the kernels' instructions and the small per-pass arrays stay in L2
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// bulk_g2s with an L2 cache policy
// dst[i] += src[i] (fp32) for bytes / 4 elements: a bulk reduction from
// shared to global memory by the copy engine (16-byte aligned, size a
// multiple of 16). The calling thread waits until the reduction has been
// performed, so the CTA may exit and the grid completes with y final.
__device__ __forceinline__ void bulk_reduce_add_f32(float *dst, const float *src, uint32_t bytes) {
    asm volatile(
        "cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
        "r"(smem_addr(src)), "r"(bytes)
        : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// generic-proxy writes to shared memory made visible to the async proxy
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
        "%2, [%3], %4;" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol)
        : "memory");
}

__device__ __forceinline__ void red_add_v4(float *dst, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

// gate activation of s = u * act(g): SiLU(g) = g / (1 + e^-g) for SwiGLU,
// GELU(g) = g (1 + erf(g / sqrt 2)) / 2 for GeGLU (CUDA's expf and erff)
__device__ __forceinline__ float gate_act(float g, int act) {
    return act == PROX_ACT_GEGLU ? 0.5f * g * (1.f + erff(g * 0.70710678118654752f))
                                 : g / (1.f + expf(-g));
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

#endif  // __CUDACC__

}  // namespace prox
