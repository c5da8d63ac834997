// Stage 2 of the Prox FFN on the tensor cores, for passes of several tokens:
// the kept channels of all the pass's tokens are gathered into one union
// list, and the exact up/gate and down projections over that union become
// small dense GEMMs (weights as the UMMA M operand, the pass's tokens as N),
// run by tcgen05.mma with fp32 accumulators in tensor memory. Each token's
// own channel mask is applied to s, so the result is the per-token
// computation of the Prox deep-dive blog, section "Stage 2" (Pi_out / Pi_in
// of the translated arXiv page, section 2.2), for every token at once. The
// pages leave batches beyond one token open (blog, "Limitations"); this is
// the plain reading: a channel kept by any token is read once per pass.
//
// Two kernels, chained with programmatic dependent launch after Stage 1:
//   k_s2u_updown: one MMA tile is 64 union channels: A rows 0..63 are their
//     W_up rows and rows 64..127 their W_gate rows (K-major), B = x over the
//     full d_model (K-major), so D holds u (lanes 0..63) and g (lanes 64..127).
//     The (tile, 64-wide K block) steps are split evenly among the CTAs as
//     contiguous ranges (stream-K); a CTA accumulates in TMEM while its steps
//     stay in one tile. A tile split between CTAs is summed in global fp32
//     with vector atomics, and the CTA that completes it forms s = u * act(g)
//     (zero where the token did not keep the channel), splits it into bf16 hi
//     + lo (s = hi + lo to about 2^-16) and stores it as ready 128-byte-
//     swizzled B tiles (one 64-position K block per tile).
//   k_s2u_down: y^T += W_down[union]^T s^T. A stage holds 32 union positions
//     x 512 (or 256) output coordinates of W_down (row-major, so each position
//     is one 1 KB run; an MN-major A operand) and the s tiles of those
//     positions; four (two) M = 128 MMAs per 16 positions, hi and lo of s into
//     one accumulator each. Steps (coordinate tile, 32 positions) are split
//     evenly among CTAs; each CTA adds its accumulated block to y with fp32
//     atomics whenever its range leaves a coordinate tile.
// Both kernels: one CTA per SM, warp-specialised (roles below); the loader
// threads move 16-byte pieces of the gathered rows with cp.async (L2
// evict-first) straight into the swizzled layout the MMA reads, one thread
// issues the MMAs, and tcgen05.commit on a per-stage mbarrier frees a stage
// for reuse. All waits are bounded; TMEM is freed before exit.
#include "prox_internal.cuh"
#include "umma.cuh"

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace prox {

namespace {

constexpr int kUM = 128;              // UMMA M
constexpr int kUN = 16;               // UMMA N: token slots (the pass's tokens, rest zero)
constexpr int kUK = 64;               // K elements per up/gate stage: one 128-byte swizzle row
constexpr int kTile = 64;             // union channels per up/gate tile (= positions per s tile)
constexpr int kDnPos = 32;            // union positions per down stage
constexpr uint32_t kAtom = 1024;      // 8 rows x 128 bytes
constexpr uint32_t kInvalid = 0xFFFFFFFFu;

// ring stage sizes (bytes, multiples of the 1024-byte swizzle atom)
constexpr uint32_t kUgStage = 16384 + 2 * kAtom;   // A (64 up + 64 gate rows) | x (16 rows)
__host__ __device__ constexpr uint32_t dn_a_bytes(int cw) { return (uint32_t)kDnPos * cw * 2; }
__host__ __device__ constexpr uint32_t dn_stage(int cw) { return dn_a_bytes(cw) + 4 * kAtom; }

// instruction descriptor of kind::f16: bf16 A and B, fp32 D, M = 128,
// N = 16, B K-major, A K-major or MN-major
__host__ __device__ constexpr uint32_t bf16_idesc(bool a_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((uint32_t)(kUN >> 3) << 17) | ((uint32_t)(kUM >> 4) << 24);
}

// 16-byte cp.async with an L2 policy; src_bytes 0 fills the 16 bytes with
// zeros and reads nothing
__device__ __forceinline__ void cp16_pol(uint32_t dst, const void *src, uint32_t src_bytes,
                                         uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst),
                 "l"(src), "r"(src_bytes), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// byte offset of 16-byte chunk `c` of row `r` in a K-major 128-byte-swizzled
// tile (8-row atoms, 1024 bytes apart)
__device__ __forceinline__ uint32_t kmaj_off(int r, int c) {
    return (uint32_t)(r >> 3) * kAtom + (uint32_t)(r & 7) * 128u +
           ((uint32_t)(c ^ (r & 7)) << 4);
}

// Bounded wait shared by all threads of the CTA: once any wait has given up,
// later ones return at once (the CTA then skips its remaining MMAs).
__device__ __forceinline__ bool cta_wait(uint64_t *bar, uint32_t parity, const Stage2UArgs &a,
                                         volatile int *fail) {
    if (*fail) return false;
    if (mbar_wait(bar, parity, a.wait_us)) return true;
    *fail = 1;
    atomicOr(a.status, kStTimeoutMma);
    return false;
}

// exclusive scan of n counts (in place, n <= 1024) by one warp; returns the total
__device__ int warp_scan_inplace(int *v, int n, int lane) {
    const int per = (n + 31) / 32;
    const int c0 = lane * per;
    int loc = 0;
    for (int k = 0; k < per; ++k)
        if (c0 + k < n) loc += v[c0 + k];
    int inc = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int m = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += m;
    }
    int run = inc - loc;
    for (int k = 0; k < per; ++k)
        if (c0 + k < n) {
            const int t = v[c0 + k];
            v[c0 + k] = run;
            run += t;
        }
    return __shfl_sync(0xffffffffu, inc, 31);
}

// ---------------------------------------------------------------------------
// shared-memory carve-up (offsets from a 1024-byte aligned base)
// ---------------------------------------------------------------------------
struct UgSmem {
    uint32_t ring, bars, misc, xg, uscan, rows, total;
};
__host__ __device__ inline UgSmem ug_smem(int nstage, int C, int span) {
    UgSmem s;
    uint32_t o = 0;
    s.ring = o;
    o += (uint32_t)nstage * kUgStage;
    s.bars = o;
    o += (uint32_t)(2 * nstage + 5) * 8;
    s.misc = o;
    o += 16;
    s.xg = o;                                      // g of a tile, handed to the u warps
    o += (uint32_t)kTile * 8 * 4;
    s.uscan = o;
    o += (uint32_t)(C + 1 > 8 ? C + 1 : 8) * 4;  // also per-token offsets at the end
    o = (o + 15) & ~15u;
    s.rows = o;
    o += (uint32_t)span * kTile * 4;
    s.total = o + 1024;  // alignment slack of the dynamic shared memory base
    return s;
}

struct DnSmem {
    uint32_t ring, bars, misc, rows, total;
};
__host__ __device__ inline DnSmem dn_smem(int nstage, int cw, int rows_cap) {
    DnSmem s;
    uint32_t o = 0;
    s.ring = o;
    o += (uint32_t)nstage * dn_stage(cw);
    s.bars = o;
    o += (uint32_t)(2 * nstage + 5) * 8;
    s.misc = o;
    o += 16;
    s.rows = o;
    o += (uint32_t)rows_cap * 4;
    s.total = o + 1024;
    return s;
}

// This CTA's share [s0, s1) of n steps split evenly over the grid
__device__ __forceinline__ void even_range(int n, int &s0, int &s1) {
    s0 = (int)((long long)n * blockIdx.x / gridDim.x);
    s1 = (int)((long long)n * (blockIdx.x + 1) / gridDim.x);
}

// Roles (both kernels): warps 0..7 load (every thread issues its share of a
// stage's 16-byte copies, then cp.async.mbarrier.arrive.noinc on the stage's
// "full" barrier, so no thread ever waits for its own copies and the whole
// ring stays in flight); warp 8 issues the MMAs (one lane) and frees stages
// with tcgen05.commit on their "empty" barriers; warps 9..12 (one per TMEM
// lane quadrant) run the epilogues from two alternating accumulators.
constexpr int kLoadWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kEpiWarp0 = 9;
constexpr int kThreads = (kEpiWarp0 + 4) * 32;

__device__ __forceinline__ void cp_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// barriers of a kernel: full[NST], empty[NST], acc_full[2], acc_empty[2],
// fin (every MMA the kernel issued is complete)
struct Bars {
    uint64_t *full, *empty, *acc_full, *acc_empty, *fin;
};
__device__ __forceinline__ Bars carve_bars(unsigned char *p, int nst) {
    uint64_t *b = reinterpret_cast<uint64_t *>(p);
    return Bars{b, b + nst, b + 2 * nst, b + 2 * nst + 2, b + 2 * nst + 4};
}
__device__ __forceinline__ void init_bars(const Bars &b, int nst) {
    for (int s = 0; s < nst; ++s) {
        mbar_init(&b.full[s], kLoadWarps * 32);
        mbar_init(&b.empty[s], 1);
    }
    for (int k = 0; k < 2; ++k) {
        mbar_init(&b.acc_full[k], 1);
        mbar_init(&b.acc_empty[k], 128);
    }
    mbar_init(b.fin, 1);
    mbar_fence_init();
}

// ---------------------------------------------------------------------------
// up/gate over the union: u, g (TMEM) -> s tiles
// ---------------------------------------------------------------------------
template <int B>
__global__ void __launch_bounds__(kThreads, 1) k_s2u_updown(const Stage2UArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int d = a.d, C = a.C, NST = a.nstage;
    const uint32_t sbase = (smem_addr(smem_raw) + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - smem_addr(smem_raw));
    const UgSmem L = ug_smem(NST, C, a.span);
    const Bars bar = carve_bars(smem + L.bars, NST);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.misc);
    volatile int *fail = reinterpret_cast<volatile int *>(smem + L.misc + 4);
    volatile int *last = reinterpret_cast<volatile int *>(smem + L.misc + 8);
    float *xg = reinterpret_cast<float *>(smem + L.xg);
    int *uscan = reinterpret_cast<int *>(smem + L.uscan);
    uint32_t *rows = reinterpret_cast<uint32_t *>(smem + L.rows);

    // token rows of the x tiles that no copy fills stay zero
    for (int s = 0; s < NST; ++s) {
        uint4 *xz = reinterpret_cast<uint4 *>(smem + L.ring + s * kUgStage + 16384);
        for (int k = tid; k < (int)(2 * kAtom / 16); k += kThreads) xz[k] = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
    if (tid == 0) {
        init_bars(bar, NST);
        *fail = 0;
    }
    if (wid == kMmaWarp) tmem_alloc(tmem_slot, 32);

    // Stage 1's lists (and its clearing of the partial sums) are complete
    // once it has finished
    if (tid == 0) stamp_min(a.stamps, kS2Entry);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    if (tid == 0) {
        stamp_min(a.stamps, kS2Go);
        stamp_max(a.stamps, kS2GoMax);
    }
    for (int c = tid; c < C; c += kThreads) uscan[c] = a.ucount[c];
    __syncthreads();
    if (wid == 0) {
        const int tot = warp_scan_inplace(uscan, C, lane);
        if (lane == 0) uscan[C] = tot;
    }
    __syncthreads();
    const int nU = uscan[C] < a.f ? uscan[C] : a.f;
    const int NKB = d / kUK;                      // K blocks per tile
    const int ntiles = (nU + kTile - 1) / kTile;
    int S0, S1;
    even_range(ntiles * NKB, S0, S1);
    const int nsteps = S1 - S0;
    const int t_lo = S0 / NKB;
    const int t_hi = nsteps > 0 ? (S1 - 1) / NKB : t_lo - 1;
    // union entries (channel | token bits << 24) of this CTA's tiles
    for (int k = tid; k < (t_hi - t_lo + 1) * kTile; k += kThreads) {
        const int tile = t_lo + k / kTile, p = tile * kTile + k % kTile;
        uint32_t e = kInvalid;
        if (p < nU) {
            int lo = 0, hi = C - 1;  // block c with uscan[c] <= p < uscan[c + 1]
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (uscan[mid] <= p) lo = mid; else hi = mid - 1;
            }
            e = a.ulist[(size_t)lo * kCB + (p - uscan[lo])];
            if ((int)(e & 0xFFFFFFu) >= a.f) e = kInvalid;  // never read outside W
            // the CTA holding the tile's first K block publishes the positions
            if (tile * NKB >= S0) a.pos_ch[p] = e;
        }
        rows[k] = e;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t ring = sbase + L.ring;

    if (wid < kLoadWarps) {
        // ---------------- loaders ----------------
        const uint64_t pol = l2_evict_first();
        const int c = tid & 7;
        for (int ls = 0; ls < nsteps; ++ls) {
            const int stg = ls % NST;
            if (ls >= NST) cta_wait(&bar.empty[stg], ((ls / NST) - 1) & 1, a, fail);
            const int step = S0 + ls;
            const int tile = step / NKB, kb = step % NKB;
            const uint32_t st = ring + (uint32_t)stg * kUgStage;
            const uint32_t *er = rows + (tile - t_lo) * kTile;
            // 64 up rows, then the same channels' gate rows, 128 bytes each
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = (tid >> 3) + 32 * j;
                const uint32_t e = er[r & (kTile - 1)];
                if (e == kInvalid) continue;  // rows past the union: never read back
                const uint16_t *w = (r < kTile) ? a.w_up : a.w_gate;
                cp16_pol(st + kmaj_off(r, c), w + (size_t)(e & 0xFFFFFFu) * d + kb * kUK + c * 8,
                         16, pol);
            }
            if (tid < B * 8) {
                const int t = tid >> 3;
                if (t < a.nb)
                    cp16(st + 16384u + kmaj_off(t, c), a.x + (size_t)t * d + kb * kUK + c * 8);
            }
            if (a.debug_skip == ls && blockIdx.x == 0) continue;  // test hook: never filled
            cp_arrive_noinc(&bar.full[stg]);
        }
        cp_wait_all();
    } else if (wid == kMmaWarp) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = bf16_idesc(false);
            int seg = 0;
            for (int s = 0; s < nsteps; ++s) {
                const int stg = s % NST;
                const int kb = (S0 + s) % NKB;
                const bool seg_first = (s == 0) || kb == 0;
                const bool seg_last = (s == nsteps - 1) || kb == NKB - 1;
                const uint32_t acc = tmem + (uint32_t)(seg & 1) * kUN;
                if (seg_first && seg >= 2) cta_wait(&bar.acc_empty[seg & 1], ((seg >> 1) - 1) & 1, a, fail);
                cta_wait(&bar.full[stg], (s / NST) & 1, a, fail);
                tc_fence_after();
                if (!*fail) {
                    const uint32_t st = ring + (uint32_t)stg * kUgStage;
#pragma unroll
                    for (int kk = 0; kk < kUK / 16; ++kk)
                        umma(acc, sw128_desc(st + kk * 32, 16, kAtom),
                             sw128_desc(st + 16384u + kk * 32, 16, kAtom), idesc,
                             (seg_first && kk == 0) ? 0u : 1u);
                }
                umma_commit(&bar.empty[stg]);
                if (seg_last) {
                    umma_commit(&bar.acc_full[seg & 1]);
                    ++seg;
                }
            }
            umma_commit(bar.fin);  // also after a failed wait: no MMA is left running
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: one segment per tile this CTA touches ----
        const int q = wid & 3;                       // TMEM lane quadrant
        const int r = q * 32 + lane;                 // A row: u (r < 64) or g
        const int et = tid - kEpiWarp0 * 32;         // 0..127
        for (int tile = t_lo, seg = 0; tile <= t_hi; ++tile, ++seg) {
            const int kb0 = (tile * NKB > S0 ? tile * NKB : S0) - tile * NKB;
            const int kb1 = ((tile + 1) * NKB < S1 ? (tile + 1) * NKB : S1) - tile * NKB;
            const bool whole = (kb0 == 0 && kb1 == NKB);
            const int p = tile * kTile + (r & (kTile - 1));
            if (!cta_wait(&bar.acc_full[seg & 1], (seg >> 1) & 1, a, fail))
                mbar_wait(bar.fin, 0, kDefaultWaitUs);  // no MMA running while TMEM is read
            tc_fence_after();
            float v[8];
            tmem_ld8(tmem + (uint32_t)(seg & 1) * kUN + ((uint32_t)(q * 32) << 16), v);
            tc_fence_before();
            mbar_arrive(&bar.acc_empty[seg & 1]);
            if (!whole) {
                if (p < nU) {
                    float *dst = a.ug + (size_t)p * 2 * B + (r < kTile ? 0 : B);
                    red_add_v4(dst, v[0], v[1], v[2], v[3]);
                    if (B == 8) red_add_v4(dst + 4, v[4], v[5], v[6], v[7]);
                    __threadfence();
                }
            } else if (r >= kTile) {
#pragma unroll
                for (int t = 0; t < 8; ++t) xg[(r - kTile) * 8 + t] = v[t];
            }
            named_bar_sync(1, 128);
            if (et == 0) {
                int l = 1;
                if (!whole) {
                    const int n = kb1 - kb0;
                    l = (atomicAdd(a.tile_cnt + tile, n) + n == NKB);
                }
                *last = l;
            }
            named_bar_sync(1, 128);
            if (*last && r < kTile) {
                // this CTA completes the tile: s = u * act(g) per kept (token,
                // channel), as bf16 hi + lo in the down GEMM's swizzled B layout
                float g[8];
                if (whole) {
#pragma unroll
                    for (int t = 0; t < 8; ++t) g[t] = xg[r * 8 + t];
                } else {
                    __threadfence();
                    if (p < nU) {
                        const float4 *src = reinterpret_cast<const float4 *>(a.ug + (size_t)p * 2 * B);
                        float4 w4 = __ldcg(src);
                        v[0] = w4.x; v[1] = w4.y; v[2] = w4.z; v[3] = w4.w;
                        if (B == 8) { w4 = __ldcg(src + 1); v[4] = w4.x; v[5] = w4.y; v[6] = w4.z; v[7] = w4.w; }
                        w4 = __ldcg(src + B / 4);
                        g[0] = w4.x; g[1] = w4.y; g[2] = w4.z; g[3] = w4.w;
                        if (B == 8) { w4 = __ldcg(src + B / 4 + 1); g[4] = w4.x; g[5] = w4.y; g[6] = w4.z; g[7] = w4.w; }
                    }
                }
                const uint32_t e = rows[(tile - t_lo) * kTile + r];
                const uint32_t bits = (p < nU) ? (e >> 24) : 0u;
                unsigned char *tb = reinterpret_cast<unsigned char *>(a.sb) + (size_t)tile * 2 * kAtom;
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    float sv = 0.f;
                    if (t < B && t < a.nb && ((bits >> t) & 1u)) sv = v[t] * gate_act(g[t], a.act);
                    const __nv_bfloat16 hi = __float2bfloat16_rn(sv);
                    const __nv_bfloat16 lo = __float2bfloat16_rn(sv - __bfloat162float(hi));
                    const uint32_t off = (uint32_t)t * 128u + ((uint32_t)((r >> 3) ^ t) << 4) + (r & 7) * 2;
                    *reinterpret_cast<__nv_bfloat16 *>(tb + off) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(tb + kAtom + off) = lo;
                }
            }
            named_bar_sync(1, 128);  // xg and *last are reused by the next tile
        }
    }

    // per-token ascending kept-channel lists and counts (blocks c = g, g + G, ...)
    __syncthreads();
    const int G = gridDim.x, gi = blockIdx.x;
    if (a.idx_s || a.count_s) {
        int *tbase = uscan;  // reused: [B] per-token offsets of block c
        for (int c = gi; c < C; c += G) {
            __syncthreads();
            if (wid < a.nb) {
                int sum = 0;
                for (int k = lane; k < c; k += 32) sum += a.tcount[k * B + wid];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (lane == 0) tbase[wid] = sum;
            }
            __syncthreads();
            if (a.idx_s)
                for (int t = 0; t < a.nb; ++t) {
                    const int nk = a.tcount[c * B + t];
                    for (int k = tid; k < nk; k += kThreads)
                        a.idx_s[(size_t)t * a.f + tbase[t] + k] = a.tlist[(size_t)t * a.f + c * kCB + k];
                }
        }
        if (gi == 0 && a.count_s && wid < a.nb) {
            int sum = 0;
            for (int k = lane; k < C; k += 32) sum += a.tcount[k * B + wid];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (lane == 0) a.count_s[wid] = sum;
        }
    }
    // tensor memory is read and freed only once every MMA issued has completed
    // (a bounded wait that gave up leaves MMAs issued before it)
    mbar_wait(bar.fin, 0, kDefaultWaitUs);
    tc_fence_before();
    __syncthreads();
    if (wid == kMmaWarp) {
        tc_fence_after();
        tmem_free(tmem, 32);
    }
}

// ---------------------------------------------------------------------------
// down over the union: y^T += W_down[union]^T (s_hi + s_lo)^T
// ---------------------------------------------------------------------------
template <int B, int NM>  // NM: 128-coordinate M tiles per stage (coordinate tile = 128 NM)
__global__ void __launch_bounds__(kThreads, 1) k_s2u_down(const Stage2UArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    constexpr int CW = NM * kUM;                 // output coordinates per stage
    constexpr uint32_t ABYTES = dn_a_bytes(CW);
    constexpr uint32_t STG = dn_stage(CW);
    constexpr uint32_t LBO = (kDnPos / 8) * kAtom;  // stride of 64-coordinate atoms
    constexpr uint32_t ACOLS = NM * kUN;           // columns of one accumulator
    constexpr uint32_t TCOLS = 2 * ACOLS < 32 ? 32 : 2 * ACOLS;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int d = a.d, C = a.C, NST = a.nstage_dn;
    const uint32_t sbase = (smem_addr(smem_raw) + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - smem_addr(smem_raw));
    const DnSmem L = dn_smem(NST, CW, a.rows_dn);
    const Bars bar = carve_bars(smem + L.bars, NST);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.misc);
    volatile int *fail = reinterpret_cast<volatile int *>(smem + L.misc + 4);
    int *ntot = reinterpret_cast<int *>(smem + L.misc + 8);
    uint32_t *rows = reinterpret_cast<uint32_t *>(smem + L.rows);

    // token rows 8..15 of the s tiles stay zero for the whole kernel
    for (int s = 0; s < NST; ++s) {
        unsigned char *bz = smem + L.ring + s * STG + ABYTES;
        for (int k = tid; k < (int)(2 * kAtom / 16); k += kThreads) {
            const int h = k / (kAtom / 16), q = k % (kAtom / 16);
            reinterpret_cast<uint4 *>(bz + h * 2 * kAtom + kAtom)[q] = make_uint4(0, 0, 0, 0);
        }
    }
    fence_async_smem();
    if (tid == 0) {
        init_bars(bar, NST);
        *fail = 0;
    }
    if (wid == kMmaWarp) tmem_alloc(tmem_slot, TCOLS);

    // the up/gate kernel's s tiles and positions are complete once it has finished
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    if (wid == 0) {
        int sum = 0;
        for (int c = lane; c < C; c += 32) sum += a.ucount[c];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) *ntot = sum;
    }
    __syncthreads();
    const int nU = *ntot < a.f ? *ntot : a.f;
    const int NPB = (nU + kDnPos - 1) / kDnPos;   // position blocks
    int S0, S1;
    even_range((d / CW) * NPB, S0, S1);
    const int nsteps = S1 - S0;
    for (int k = tid; k < nsteps * kDnPos; k += kThreads) {
        const int p = ((S0 + k / kDnPos) % NPB) * kDnPos + k % kDnPos;
        rows[k] = p < nU ? __ldcg(a.pos_ch + p) : kInvalid;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t ring = sbase + L.ring;

    if (wid < kLoadWarps) {
        // ---------------- loaders ----------------
        const uint64_t pol = l2_evict_first();
        const unsigned char *sbg = reinterpret_cast<const unsigned char *>(a.sb);
        constexpr int CPR = CW / 8;               // 16-byte pieces per position
        for (int ls = 0; ls < nsteps; ++ls) {
            const int stg = ls % NST;
            if (ls >= NST) cta_wait(&bar.empty[stg], ((ls / NST) - 1) & 1, a, fail);
            const int step = S0 + ls;
            const int mt = step / NPB, pb = step % NPB;
            const uint32_t st = ring + (uint32_t)stg * STG;
            const uint32_t *er = rows + ls * kDnPos;
            // 32 positions x CW coordinates of W_down: each position one
            // contiguous 2 CW-byte run; MN-major, 64 coordinates per 128-byte
            // row, 8 positions per atom
#pragma unroll
            for (int i = 0; i < kDnPos * CPR / (kLoadWarps * 32); ++i) {
                const int qq = tid + kLoadWarps * 32 * i;
                const int row = qq / CPR, c = qq % CPR;
                const uint32_t e = er[row];
                const bool ok = e != kInvalid && (int)(e & 0xFFFFFFu) < a.f;
                const uint16_t *src =
                    ok ? a.w_down + (size_t)(e & 0xFFFFFFu) * d + mt * CW + c * 8 : a.w_down;
                const uint32_t off = (uint32_t)(c >> 3) * LBO + (uint32_t)(row >> 3) * kAtom +
                                     (uint32_t)(row & 7) * 128u + ((uint32_t)((c & 7) ^ (row & 7)) << 4);
                cp16_pol(st + off, src, ok ? 16u : 0u, pol);
            }
            if (tid < 128) {  // s hi and lo atoms (token rows 0..7) of the 64-position block
                const int h = tid >> 6, qq = tid & 63;
                cp16(st + ABYTES + (uint32_t)h * 2 * kAtom + qq * 16,
                     sbg + (size_t)(pb >> 1) * 2 * kAtom + h * kAtom + qq * 16);
            }
            cp_arrive_noinc(&bar.full[stg]);
        }
        cp_wait_all();
    } else if (wid == kMmaWarp) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = bf16_idesc(true);
            int seg = 0;
            for (int s = 0; s < nsteps; ++s) {
                const int stg = s % NST;
                const int pb = (S0 + s) % NPB;
                const bool seg_first = (s == 0) || pb == 0;
                const bool seg_last = (s == nsteps - 1) || pb == NPB - 1;
                const uint32_t acc = tmem + (uint32_t)(seg & 1) * ACOLS;
                if (seg_first && seg >= 2) cta_wait(&bar.acc_empty[seg & 1], ((seg >> 1) - 1) & 1, a, fail);
                cta_wait(&bar.full[stg], (s / NST) & 1, a, fail);
                tc_fence_after();
                if (!*fail) {
                    const uint32_t st = ring + (uint32_t)stg * STG;
#pragma unroll
                    for (int kk = 0; kk < kDnPos / 16; ++kk) {
                        const uint32_t bo = st + ABYTES + (uint32_t)((pb & 1) * 2 + kk) * 32;
                        const uint64_t dbh = sw128_desc(bo, 16, kAtom);
                        const uint64_t dbl = sw128_desc(bo + 2 * kAtom, 16, kAtom);
#pragma unroll
                        for (int mi = 0; mi < NM; ++mi) {
                            const uint64_t da = sw128_desc(st + mi * 2 * LBO + kk * 2 * kAtom, LBO, kAtom);
                            umma(acc + mi * kUN, da, dbh, idesc, (seg_first && kk == 0) ? 0u : 1u);
                            umma(acc + mi * kUN, da, dbl, idesc, 1u);
                        }
                    }
                }
                umma_commit(&bar.empty[stg]);
                if (seg_last) {
                    umma_commit(&bar.acc_full[seg & 1]);
                    ++seg;
                }
            }
            umma_commit(bar.fin);  // also after a failed wait: no MMA is left running
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: y += one coordinate tile's block ----------
        const int q = wid & 3;
        int seg = 0;
        for (int s = 0; s < nsteps; ++s) {
            const int step = S0 + s;
            const int pb = step % NPB;
            if (!(s == nsteps - 1 || pb == NPB - 1)) continue;
            const int mt = step / NPB;
            if (!cta_wait(&bar.acc_full[seg & 1], (seg >> 1) & 1, a, fail))
                mbar_wait(bar.fin, 0, kDefaultWaitUs);  // no MMA running while TMEM is read
            tc_fence_after();
            float D[NM][8];
#pragma unroll
            for (int mi = 0; mi < NM; ++mi)
                tmem_ld8(tmem + (uint32_t)(seg & 1) * ACOLS + mi * kUN + ((uint32_t)(q * 32) << 16), D[mi]);
            tc_fence_before();
            mbar_arrive(&bar.acc_empty[seg & 1]);
#pragma unroll
            for (int mi = 0; mi < NM; ++mi) {
                const int m = mt * CW + mi * kUM + q * 32 + lane;
#pragma unroll
                for (int t = 0; t < B; ++t)
                    if (t < a.nb) atomicAdd(a.y + (size_t)t * d + m, D[mi][t]);
            }
            ++seg;
        }
    }
    mbar_wait(bar.fin, 0, kDefaultWaitUs);
    tc_fence_before();
    __syncthreads();
    if (wid == kMmaWarp) {
        tc_fence_after();
        tmem_free(tmem, TCOLS);
    }
    if (tid == 0) stamp_max(a.stamps, kS2End);
}

template <int B, int NM>
cudaError_t launch_u(const Stage2UArgs &a, int grid, cudaStream_t s) {
    const size_t sm_ug = ug_smem(a.nstage, a.C, a.span).total;
    const size_t sm_dn = dn_smem(a.nstage_dn, NM * kUM, a.rows_dn).total;
    cudaError_t e = set_max_dynamic_smem((const void *)k_s2u_updown<B>, sm_ug);
    if (e == cudaSuccess) e = set_max_dynamic_smem((const void *)k_s2u_down<B, NM>, sm_dn);
    if (e == cudaSuccess) e = launch_pdl(k_s2u_updown<B>, dim3(grid), dim3(kThreads), sm_ug, s, a);
    if (e == cudaSuccess) e = launch_pdl(k_s2u_down<B, NM>, dim3(grid), dim3(kThreads), sm_dn, s, a);
    return e;
}

}  // namespace

// Launch plan of the tensor-core Stage 2; false if the shape is outside it
bool stage2u_plan(int d, int f, int num_sms, Stage2UPlan *p) {
    const int C = f / kCB;
    const int nkb = d / kUK;
    const int stepsA = (f / kTile) * nkb;                       // at most
    const int lenA = (stepsA + num_sms - 1) / num_sms;
    p->span = (lenA + nkb - 1) / nkb + 1;
    p->cw = (d % 512 == 0) ? 512 : 256;
    const int stepsB = (d / p->cw) * ((f + kDnPos - 1) / kDnPos);
    p->rows_dn = (stepsB + num_sms - 1) / num_sms * kDnPos;
    const size_t budget = (size_t)kS2SmemBudget;
    int na = 12, nb = 8;
    while (na > 0 && ug_smem(na, C, p->span).total > budget) --na;
    while (nb > 0 && dn_smem(nb, p->cw, p->rows_dn).total > budget) --nb;
    p->nstage = na;
    p->nstage_dn = nb;
    return na >= 4 && nb >= 3;
}

cudaError_t launch_stage2_umma(int B, const Stage2UArgs &a, int grid, cudaStream_t s) {
    if (a.cw == 512) {
        if (B == 4) return launch_u<4, 4>(a, grid, s);
        if (B == 8) return launch_u<8, 4>(a, grid, s);
    } else if (a.cw == 256) {
        if (B == 4) return launch_u<4, 2>(a, grid, s);
        if (B == 8) return launch_u<8, 2>(a, grid, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace prox
