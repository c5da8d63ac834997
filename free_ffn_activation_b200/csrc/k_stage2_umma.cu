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
//   k_s2u_updown: U = W_up[union] x^T and G = W_gate[union] x^T over the full
//     x, M = 128 union channels per tile, K = d_model split into ks slices.
//     A CTA takes a contiguous range of (tile, slice) units and accumulates
//     consecutive slices of one tile in TMEM; partial tiles are summed in
//     global fp32 with vector atomics, and the CTA that completes a tile forms
//     s = u * act(g) (zero where the token did not keep the channel), splits it
//     into bf16 hi + lo (s = hi + lo to about 2^-16) and stores it as ready
//     128-byte-swizzled B tiles.
//   k_s2u_down: y^T += W_down[union]^T s^T, M = 128 d_model coordinates, K =
//     union positions (W_down is row-major, so the A tile is MN-major), N =
//     tokens; the hi and lo halves of s are two MMAs into one accumulator.
//     Units (position range, coordinate tile) go to CTAs in contiguous ranges;
//     each unit adds its 128 x nb block to y with fp32 atomics.
// Both kernels: 256 threads, one CTA per SM; every thread moves 16-byte
// pieces of the gathered rows with cp.async (L2 evict-first) straight into
// the swizzled layout the MMA reads, one thread issues the MMAs, and
// tcgen05.commit on a per-stage mbarrier frees a stage for reuse. All waits
// are bounded; TMEM (32 columns) is freed before exit.
#include "prox_internal.cuh"

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace prox {

namespace {

constexpr int kUT = 256;              // threads per CTA
constexpr int kUM = 128;              // UMMA M
constexpr int kUN = 16;               // UMMA N: token slots (the pass's tokens, rest zero)
constexpr int kUK = 64;               // K elements per stage: one 128-byte swizzle row of bf16
constexpr uint32_t kAtom = 1024;      // 8 rows x 128 bytes
constexpr uint32_t kInvalid = 0xFFFFFFFFu;
constexpr int kTmemCols = 32;

// ring stage sizes (bytes, multiples of the 1024-byte swizzle atom)
constexpr uint32_t kUgStage = 2 * 16384 + 2 * kAtom;   // A_up | A_gate | x (16 rows)
constexpr uint32_t kDnStage = 16384 + 4 * kAtom;       // A_down | s hi (16 rows) | s lo (16 rows)

// ---------------------------------------------------------------------------
// tcgen05 / UMMA helpers
// ---------------------------------------------------------------------------
// shared-memory matrix descriptor of a 128-byte-swizzled tile: start address,
// leading and stride byte offsets in 16-byte units, descriptor version 1,
// layout type 2 (128-byte swizzle)
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// instruction descriptor of kind::f16: bf16 A and B, fp32 D, M = 128,
// N = 16, B K-major, A K-major or MN-major
__host__ __device__ constexpr uint32_t bf16_idesc(bool a_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((uint32_t)(kUN >> 3) << 17) | ((uint32_t)(kUM >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t da, uint64_t db, uint32_t idesc,
                                     uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(da), "l"(db), "r"(idesc), "r"(accumulate)
        : "memory");
}

// arrive on `bar` once every MMA this thread issued so far has completed
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// generic-proxy writes to shared memory (cp.async, st.shared) made visible to
// the tensor core's async-proxy reads
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 8 consecutive fp32 columns of this thread's TMEM lane (warp w reads lanes
// 32 (w % 4) .. + 31); load and wait in one statement so no use of the
// registers can be scheduled before the wait
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r0, r1, r2, r3, r4, r5, r6, r7;
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3), "=r"(r4), "=r"(r5), "=r"(r6), "=r"(r7)
        : "r"(taddr)
        : "memory");
    v[0] = __uint_as_float(r0);
    v[1] = __uint_as_float(r1);
    v[2] = __uint_as_float(r2);
    v[3] = __uint_as_float(r3);
    v[4] = __uint_as_float(r4);
    v[5] = __uint_as_float(r5);
    v[6] = __uint_as_float(r6);
    v[7] = __uint_as_float(r7);
}

// TMEM allocation by one whole warp; the address lands in *slot
__device__ __forceinline__ void tmem_alloc(uint32_t *slot) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_free(uint32_t taddr) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
                 "r"(kTmemCols)
                 : "memory");
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
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_wait_dyn(int n) {
    // the ring depth is a launch parameter; wait_group takes an immediate
    switch (n) {
        case 0: cp_wait<0>(); break;
        case 1: cp_wait<1>(); break;
        case 2: cp_wait<2>(); break;
        case 3: cp_wait<3>(); break;
        case 4: cp_wait<4>(); break;
        case 5: cp_wait<5>(); break;
        case 6: cp_wait<6>(); break;
        case 7: cp_wait<7>(); break;
        case 8: cp_wait<8>(); break;
        default: cp_wait<9>(); break;
    }
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
    uint32_t ring, bars, misc, uscan, rows, total;
};
__host__ __device__ inline UgSmem ug_smem(int nstage, int C, int span) {
    UgSmem s;
    uint32_t o = 0;
    s.ring = o;
    o += (uint32_t)nstage * kUgStage;
    s.bars = o;
    o += (uint32_t)(nstage + 1) * 8;
    s.misc = o;
    o += 16;
    s.uscan = o;
    o += (uint32_t)(C + 1 > 8 ? C + 1 : 8) * 4;  // also per-token offsets at the end
    o = (o + 15) & ~15u;
    s.rows = o;
    o += (uint32_t)span * kUM * 4;
    s.total = o + 1024;  // alignment slack of the dynamic shared memory base
    return s;
}

struct DnSmem {
    uint32_t ring, bars, misc, rows, total;
};
__host__ __device__ inline DnSmem dn_smem(int nstage, int span) {
    DnSmem s;
    uint32_t o = 0;
    s.ring = o;
    o += (uint32_t)nstage * kDnStage;
    s.bars = o;
    o += (uint32_t)(nstage + 1) * 8;
    s.misc = o;
    o += 16;
    s.rows = o;
    o += (uint32_t)span * kUnitPos * 4;
    s.total = o + 1024;
    return s;
}

// ---------------------------------------------------------------------------
// up/gate over the union: U, G (TMEM) -> s tiles
// ---------------------------------------------------------------------------
template <int B>
__global__ void __launch_bounds__(kUT, 1) k_s2u_updown(const Stage2UArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int d = a.d, C = a.C, KS = a.ks, NST = a.nstage;
    const uint32_t sbase = (smem_addr(smem_raw) + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - smem_addr(smem_raw));
    const UgSmem L = ug_smem(NST, C, a.span);
    uint64_t *bar_free = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *bar_acc = bar_free + NST;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.misc);
    volatile int *fail = reinterpret_cast<volatile int *>(smem + L.misc + 4);
    volatile int *last = reinterpret_cast<volatile int *>(smem + L.misc + 8);
    int *uscan = reinterpret_cast<int *>(smem + L.uscan);
    uint32_t *rows = reinterpret_cast<uint32_t *>(smem + L.rows);

    // the x tiles' unused token rows stay zero for the whole kernel
    for (int s = 0; s < NST; ++s) {
        uint4 *xz = reinterpret_cast<uint4 *>(smem + L.ring + s * kUgStage + 2 * 16384);
        for (int k = tid; k < (int)(2 * kAtom / 16); k += kUT) xz[k] = make_uint4(0, 0, 0, 0);
    }
    if (tid == 0) {
        for (int s = 0; s <= NST; ++s) mbar_init(&bar_free[s], 1);
        *fail = 0;
        mbar_fence_init();
    }
    if (wid == 0) tmem_alloc(tmem_slot);

    // Stage 1's lists (and its clearing of the partial sums) are complete
    // once it has finished
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    for (int c = tid; c < C; c += kUT) uscan[c] = a.ucount[c];
    __syncthreads();
    if (wid == 0) {
        const int tot = warp_scan_inplace(uscan, C, lane);
        if (lane == 0) uscan[C] = tot;
    }
    __syncthreads();
    const int nU = uscan[C] < a.f ? uscan[C] : a.f;
    const int ntiles = (nU + kUM - 1) / kUM;
    const int nunits = ntiles * KS;
    const int G = gridDim.x, g = blockIdx.x;
    const int u0 = (int)((long long)nunits * g / G), u1 = (int)((long long)nunits * (g + 1) / G);
    const int t_lo = u0 / KS;
    // union entries (channel | token bits << 24) of this CTA's tiles
    if (u1 > u0) {
        const int t_hi = (u1 - 1) / KS;
        for (int k = tid; k < (t_hi - t_lo + 1) * kUM; k += kUT) {
            const int tile = t_lo + k / kUM, p = tile * kUM + k % kUM;
            uint32_t e = kInvalid;
            if (p < nU) {
                int lo = 0, hi = C - 1;  // block c with uscan[c] <= p < uscan[c + 1]
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (uscan[mid] <= p) lo = mid; else hi = mid - 1;
                }
                e = a.ulist[(size_t)lo * kCB + (p - uscan[lo])];
                if ((int)(e & 0xFFFFFFu) >= a.f) e = kInvalid;  // never read outside W
                // the CTA holding the tile's first slice publishes the positions
                if (tile * KS >= u0) a.pos_ch[p] = e;
            }
            rows[k] = e;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int kbpu = d / kUK / KS;  // K blocks per unit
    const int nsteps = (u1 - u0) * kbpu;
    const uint64_t pol = l2_evict_first();
    const uint32_t ring = sbase + L.ring;
    constexpr uint32_t idesc = bf16_idesc(false);

    // issue the copies of step ls into its ring stage
    auto load = [&](int ls) {
        const int u = u0 + ls / kbpu;
        const int tile = u / KS, kb = (u % KS) * kbpu + ls % kbpu;
        const uint32_t st = ring + (uint32_t)(ls % NST) * kUgStage;
        const uint32_t *er = rows + (tile - t_lo) * kUM;
        const int c = tid & 7;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = (tid >> 3) + 32 * (j & 3);
            const uint32_t e = er[r];
            if (e == kInvalid) continue;  // rows past the union: never read back
            const uint16_t *w = (j < 4) ? a.w_up : a.w_gate;
            cp16_pol(st + (uint32_t)(j >> 2) * 16384u + kmaj_off(r, c),
                     w + (size_t)(e & 0xFFFFFFu) * d + kb * kUK + c * 8, 16, pol);
        }
        if (tid < B * 8) {
            const int t = tid >> 3;
            if (t < a.nb) cp16(st + 2 * 16384u + kmaj_off(t, c), a.x + (size_t)t * d + kb * kUK + c * 8);
        }
    };

    for (int ls = 0; ls < NST - 1; ++ls) {
        if (ls < nsteps) load(ls);
        cp_commit();
    }
    int nseg = 0;
    for (int s = 0; s < nsteps; ++s) {
        const int u = u0 + s / kbpu, j = s % kbpu;
        const int tile = u / KS;
        const bool seg_first = (s == 0) || (j == 0 && (u % KS) == 0);
        const bool seg_last = (s == nsteps - 1) || (j == kbpu - 1 && ((u + 1) % KS) == 0);
        const int stg = s % NST;
        cp_wait_dyn(NST - 2);
        fence_async_smem();
        __syncthreads();
        if (tid == 0 && !*fail) {
            tc_fence_after();
            const uint32_t st = ring + (uint32_t)stg * kUgStage;
#pragma unroll
            for (int kk = 0; kk < kUK / 16; ++kk) {
                const uint64_t db = sw128_desc(st + 2 * 16384u + kk * 32, 16, kAtom);
                const uint32_t acc = (seg_first && kk == 0) ? 0u : 1u;
                umma(tmem, sw128_desc(st + kk * 32, 16, kAtom), db, idesc, acc);
                umma(tmem + 16, sw128_desc(st + 16384u + kk * 32, 16, kAtom), db, idesc, acc);
            }
            umma_commit(&bar_free[stg]);
            if (seg_last) umma_commit(bar_acc);
        }
        // refill the stage step s - 1 used, once its MMAs are done
        if (s >= 1) cta_wait(&bar_free[(s - 1) % NST], ((s - 1) / NST) & 1, a, fail);
        if (s + NST - 1 < nsteps) load(s + NST - 1);
        cp_commit();

        if (!seg_last) continue;
        // ---- epilogue of a tile segment: slices [ks_lo, ks_hi) of `tile`
        const int ks_lo = (tile * KS > u0 ? tile * KS : u0) - tile * KS;
        const int ks_hi = u + 1 - tile * KS;
        const bool whole = (ks_lo == 0 && ks_hi == KS);
        cta_wait(bar_acc, nseg & 1, a, fail);
        ++nseg;
        tc_fence_after();
        const int r = (wid & 3) * 32 + lane;
        const int p = tile * kUM + r;
        float U[8], Gt[8];
        if (wid < 4) {
            const uint32_t ta = tmem + ((uint32_t)(wid * 32) << 16);
            tmem_ld8(ta, U);
            tmem_ld8(ta + 16, Gt);
            if (!whole && p < nU) {
                float *dst = a.ug + (size_t)p * 2 * B;
                red_add_v4(dst, U[0], U[1], U[2], U[3]);
                if (B == 8) red_add_v4(dst + 4, U[4], U[5], U[6], U[7]);
                red_add_v4(dst + B, Gt[0], Gt[1], Gt[2], Gt[3]);
                if (B == 8) red_add_v4(dst + B + 4, Gt[4], Gt[5], Gt[6], Gt[7]);
                __threadfence();
            }
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            int l = 1;
            if (!whole) {
                const int n = ks_hi - ks_lo;
                l = (atomicAdd(a.tile_cnt + tile, n) + n == KS);
            }
            *last = l;
        }
        __syncthreads();
        if (*last && wid < 4) {
            // this CTA completes the tile: s = u * act(g) per kept (token,
            // channel), as bf16 hi + lo in the down GEMM's swizzled B layout
            if (!whole) {
                __threadfence();
                if (p < nU) {
                    const float4 *src = reinterpret_cast<const float4 *>(a.ug + (size_t)p * 2 * B);
                    float4 v = __ldcg(src);
                    U[0] = v.x; U[1] = v.y; U[2] = v.z; U[3] = v.w;
                    if (B == 8) { v = __ldcg(src + 1); U[4] = v.x; U[5] = v.y; U[6] = v.z; U[7] = v.w; }
                    v = __ldcg(src + B / 4);
                    Gt[0] = v.x; Gt[1] = v.y; Gt[2] = v.z; Gt[3] = v.w;
                    if (B == 8) { v = __ldcg(src + B / 4 + 1); Gt[4] = v.x; Gt[5] = v.y; Gt[6] = v.z; Gt[7] = v.w; }
                }
            }
            const uint32_t e = rows[(tile - t_lo) * kUM + r];
            const uint32_t bits = (p < nU) ? (e >> 24) : 0u;
            unsigned char *tb = reinterpret_cast<unsigned char *>(a.sb) + (size_t)(p >> 6) * 2 * kAtom;
            const int kk = p & 63;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                float sv = 0.f;
                if (t < B && t < a.nb && ((bits >> t) & 1u)) sv = U[t] * gate_act(Gt[t], a.act);
                const __nv_bfloat16 hi = __float2bfloat16_rn(sv);
                const __nv_bfloat16 lo = __float2bfloat16_rn(sv - __bfloat162float(hi));
                const uint32_t off = (uint32_t)t * 128u + ((uint32_t)((kk >> 3) ^ t) << 4) + (kk & 7) * 2;
                *reinterpret_cast<__nv_bfloat16 *>(tb + off) = hi;
                *reinterpret_cast<__nv_bfloat16 *>(tb + kAtom + off) = lo;
            }
        }
    }
    cp_wait<0>();

    // per-token ascending kept-channel lists and counts (blocks c = g, g + G, ...)
    if (a.idx_s || a.count_s) {
        int *tbase = uscan;  // reused: [B] per-token offsets of block c
        for (int c = g; c < C; c += G) {
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
                    for (int k = tid; k < nk; k += kUT)
                        a.idx_s[(size_t)t * a.f + tbase[t] + k] = a.tlist[(size_t)t * a.f + c * kCB + k];
                }
        }
        if (g == 0 && a.count_s && wid < a.nb) {
            int sum = 0;
            for (int k = lane; k < C; k += 32) sum += a.tcount[k * B + wid];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (lane == 0) a.count_s[wid] = sum;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (wid == 0) {
        tc_fence_after();
        tmem_free(tmem);
    }
}

// ---------------------------------------------------------------------------
// down over the union: y^T += W_down[union]^T (s_hi + s_lo)^T
// ---------------------------------------------------------------------------
template <int B>
__global__ void __launch_bounds__(kUT, 1) k_s2u_down(const Stage2UArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int d = a.d, C = a.C, NST = a.nstage_dn;
    const uint32_t sbase = (smem_addr(smem_raw) + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - smem_addr(smem_raw));
    const DnSmem L = dn_smem(NST, a.span_dn);
    uint64_t *bar_free = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *bar_acc = bar_free + NST;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.misc);
    volatile int *fail = reinterpret_cast<volatile int *>(smem + L.misc + 4);
    int *ntot = reinterpret_cast<int *>(smem + L.misc + 8);
    uint32_t *rows = reinterpret_cast<uint32_t *>(smem + L.rows);

    // the s tiles' token rows 8..15 stay zero for the whole kernel
    for (int s = 0; s < NST; ++s) {
        unsigned char *bz = smem + L.ring + s * kDnStage + 16384;
        for (int k = tid; k < (int)(2 * kAtom / 16); k += kUT) {
            const int h = k / (kAtom / 16), q = k % (kAtom / 16);
            reinterpret_cast<uint4 *>(bz + h * 2 * kAtom + kAtom)[q] = make_uint4(0, 0, 0, 0);
        }
    }
    if (tid == 0) {
        for (int s = 0; s <= NST; ++s) mbar_init(&bar_free[s], 1);
        *fail = 0;
        mbar_fence_init();
    }
    if (wid == 0) tmem_alloc(tmem_slot);

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
    const int MT = d / kUM;
    constexpr int KPB = kUnitPos / kUK;             // K blocks per unit
    const int nkb_all = (nU + kUK - 1) / kUK;       // K blocks holding union positions
    const int NKR = (nU + kUnitPos - 1) / kUnitPos;
    const int nunits = NKR * MT;
    const int G = gridDim.x, g = blockIdx.x;
    const int u0 = (int)((long long)nunits * g / G), u1 = (int)((long long)nunits * (g + 1) / G);
    const int kr_lo = u0 / MT;
    if (u1 > u0) {
        const int kr_hi = (u1 - 1) / MT;
        for (int k = tid; k < (kr_hi - kr_lo + 1) * kUnitPos; k += kUT) {
            const int p = kr_lo * kUnitPos + k;
            rows[k] = p < nU ? __ldcg(a.pos_ch + p) : kInvalid;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t pol = l2_evict_first();
    const uint32_t ring = sbase + L.ring;
    constexpr uint32_t idesc = bf16_idesc(true);
    const unsigned char *sbg = reinterpret_cast<const unsigned char *>(a.sb);

    auto nkb = [&](int u) {
        const int r = nkb_all - (u / MT) * KPB;
        return r < KPB ? r : KPB;
    };
    // issue the copies of (unit u, K block j) into ring stage stg
    auto load = [&](int u, int j, int stg) {
        const int kr = u / MT, mt = u % MT;
        const int kb = kr * KPB + j;
        const uint32_t st = ring + (uint32_t)stg * kDnStage;
        const uint32_t *er = rows + (kr - kr_lo) * kUnitPos + j * kUK;
        const int c = tid & 15;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int row = (tid >> 4) + 16 * i;  // union position within the block (K)
            const uint32_t e = er[row];
            const bool ok = e != kInvalid && (int)(e & 0xFFFFFFu) < a.f;
            const uint16_t *src = ok ? a.w_down + (size_t)(e & 0xFFFFFFu) * d + mt * kUM + c * 8 : a.w_down;
            // MN-major: 64 coordinates per 128-byte row, 8 positions per atom
            const uint32_t off = (uint32_t)(c >> 3) * (8 * kAtom) + (uint32_t)(row >> 3) * kAtom +
                                 (uint32_t)(row & 7) * 128u + ((uint32_t)((c & 7) ^ (row & 7)) << 4);
            cp16_pol(st + off, src, ok ? 16u : 0u, pol);
        }
        if (tid < 128) {  // s hi and lo atoms (token rows 0..7), stored pre-swizzled
            const int h = tid >> 6, q = tid & 63;
            cp16(st + 16384u + (uint32_t)h * 2 * kAtom + q * 16,
                 sbg + (size_t)kb * 2 * kAtom + h * kAtom + q * 16);
        }
    };

    // loader cursor runs NST - 1 steps ahead of the consumer cursor
    int lu = u0, lj = 0, ln = 0;
    auto load_next = [&]() {
        if (lu < u1) {
            load(lu, lj, ln % NST);
            if (++lj == nkb(lu)) { ++lu; lj = 0; }
            ++ln;
        }
        cp_commit();
    };
    for (int k = 0; k < NST - 1; ++k) load_next();
    int cu = u0, cj = 0, n = 0, nseg = 0;
    while (cu < u1) {
        const int stg = n % NST;
        const bool unit_last = (cj + 1 == nkb(cu));
        cp_wait_dyn(NST - 2);
        fence_async_smem();
        __syncthreads();
        if (tid == 0 && !*fail) {
            tc_fence_after();
            const uint32_t st = ring + (uint32_t)stg * kDnStage;
#pragma unroll
            for (int kk = 0; kk < kUK / 16; ++kk) {
                const uint64_t da = sw128_desc(st + kk * 2 * kAtom, 8 * kAtom, kAtom);
                umma(tmem, da, sw128_desc(st + 16384u + kk * 32, 16, kAtom), idesc,
                     (cj == 0 && kk == 0) ? 0u : 1u);
                umma(tmem, da, sw128_desc(st + 16384u + 2 * kAtom + kk * 32, 16, kAtom), idesc, 1u);
            }
            umma_commit(&bar_free[stg]);
            if (unit_last) umma_commit(bar_acc);
        }
        if (n >= 1) cta_wait(&bar_free[(n - 1) % NST], ((n - 1) / NST) & 1, a, fail);
        load_next();
        if (unit_last) {
            cta_wait(bar_acc, nseg & 1, a, fail);
            ++nseg;
            tc_fence_after();
            if (wid < 4) {
                float D[8];
                tmem_ld8(tmem + ((uint32_t)(wid * 32) << 16), D);
                const int m = (cu % MT) * kUM + wid * 32 + lane;
#pragma unroll
                for (int t = 0; t < B; ++t)
                    if (t < a.nb) atomicAdd(a.y + (size_t)t * d + m, D[t]);
            }
            tc_fence_before();
            ++cu;
            cj = 0;
        } else {
            ++cj;
        }
        ++n;
    }
    cp_wait<0>();
    tc_fence_before();
    __syncthreads();
    if (wid == 0) {
        tc_fence_after();
        tmem_free(tmem);
    }
}

template <typename K>
cudaError_t set_smem(K k, size_t smem, size_t &configured) {
    if (smem > configured) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured = smem;
    }
    return cudaSuccess;
}

template <int B>
cudaError_t launch_u(const Stage2UArgs &a, int grid, cudaStream_t s) {
    static size_t cfg_ug = 0, cfg_dn = 0;
    const size_t sm_ug = ug_smem(a.nstage, a.C, a.span).total;
    const size_t sm_dn = dn_smem(a.nstage_dn, a.span_dn).total;
    cudaError_t e = set_smem(k_s2u_updown<B>, sm_ug, cfg_ug);
    if (e == cudaSuccess) e = set_smem(k_s2u_down<B>, sm_dn, cfg_dn);
    if (e == cudaSuccess) e = launch_pdl(k_s2u_updown<B>, dim3(grid), dim3(kUT), sm_ug, s, a);
    if (e == cudaSuccess) e = launch_pdl(k_s2u_down<B>, dim3(grid), dim3(kUT), sm_dn, s, a);
    return e;
}

}  // namespace

// Launch plan of the tensor-core Stage 2; false if the shape is outside it
bool stage2u_plan(int d, int f, int num_sms, Stage2UPlan *p) {
    const int kblocks = d / kUK;
    int ks = 8;
    while (ks > 1 && kblocks % ks) ks >>= 1;
    const int C = f / kCB;
    const int ntiles_max = f / kUM;
    const int lenA = (ntiles_max * ks + num_sms - 1) / num_sms;  // units per CTA, at most
    p->ks = ks;
    p->span = (lenA + ks - 1) / ks + 1;
    const int MT = d / kUM;
    const int nkr_max = (f + kUnitPos - 1) / kUnitPos;
    const int lenB = (nkr_max * MT + num_sms - 1) / num_sms;
    p->span_dn = (lenB + MT - 1) / MT + 1;
    const size_t budget = (size_t)kS2SmemBudget;
    const size_t fixA = ug_smem(0, C, p->span).total, fixB = dn_smem(0, p->span_dn).total;
    if (fixA >= budget || fixB >= budget) return false;
    int na = (int)((budget - fixA) / kUgStage), nb = (int)((budget - fixB) / kDnStage);
    if (na > 8) na = 8;
    if (nb > 10) nb = 10;
    p->nstage = na;
    p->nstage_dn = nb;
    return na >= 3 && nb >= 3;
}

cudaError_t launch_stage2_umma(int B, const Stage2UArgs &a, int grid, cudaStream_t s) {
    if (B == 4) return launch_u<4>(a, grid, s);
    if (B == 8) return launch_u<8>(a, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace prox
