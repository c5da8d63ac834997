// Stage 2 of the Prox sparse SwiGLU FFN on sm_100a: exact output-sparse
// up/gate over the kept channels, SiLU-mul, and the input-sparse down
// projection over the same channels (Prox deep-dive blog, section "Stage 2";
// Pi_out / Pi_in of the translated arXiv page, section 2.2; the weighted-sum
// view y = sum_j s_j W_down[j, :] of the blog's first section).
//
// One persistent CTA per SM takes an equal share of the kept channels (the
// union over the pass's tokens, in ascending order). W_up and W_gate are
// stored channel-major and W_down row-major, so a kept channel j is three
// contiguous d_model-long bf16 rows. Roles inside the CTA:
//   * a producer lane moves each channel's three rows with 1-D bulk copies
//     (TMA) into a ring of shared-memory stages (mbarrier "full");
//   * 8 dot warps take whole channels (ring slot s belongs to warp s % 8): a
//     warp forms x . W_up[j]
//     and x . W_gate[j] over the full row, reduces across its lanes, computes
//     s_j = u_j * SiLU(g_j) in fp32 and publishes it (mbarrier "sready");
//   * the down warps own fixed column slices of y: for every channel, in
//     order, they add s_j * W_down[j, slice] to register accumulators.
// A stage is refilled once its dot warp and every down warp have released it
// (mbarrier "empty"). Channels never wait on each other through a CTA-wide
// barrier, so several channels are in flight at once, and every wait is
// bounded. At the end each CTA adds its partial y to global memory with one
// bulk reduction of the copy engine.
#include "prox_internal.cuh"

#include <cuda_runtime.h>
#include <cstdint>

namespace prox {

constexpr int kNDot = 8;

// warps and shared x precision per tokens-per-pass
__host__ __device__ constexpr int s2_ndown(int B) { return B <= 2 ? 8 : 16; }
__host__ __device__ constexpr int s2_threads(int B) { return (kNDot + s2_ndown(B) + 1) * 32; }
__host__ __device__ constexpr int s2_xbytes(int B) { return (void)B, 2; }  // x as bf16

// shared-memory carve-up, shared by the kernel and the host plan
constexpr int kS2Prefetch = 4;  // channel-list blocks fetched with the counts

struct S2Smem {
    size_t stages, xs, full, empty, sready, meta, svals, uscan, tscan, chan, chanpf, total;
};

__host__ __device__ inline S2Smem s2_smem(int d, int B, int nstage, int C, int max_ch) {
    S2Smem s;
    size_t o = 0;
    s.stages = o;
    o += (size_t)nstage * 3 * d * 2;
    s.xs = o;
    o += (size_t)B * d * s2_xbytes(B);
    o = (o + 15) & ~(size_t)15;
    s.full = o;
    o += (size_t)nstage * 8;
    s.empty = o;
    o += (size_t)nstage * 8;
    s.sready = o;
    o += (size_t)nstage * 8;
    s.meta = o;
    o += (size_t)nstage * 4;
    s.svals = o;
    o += (size_t)nstage * B * 4;
    o = (o + 15) & ~(size_t)15;
    s.uscan = o;
    o += (size_t)(C + 1) * 4;
    s.tscan = o;
    o += (size_t)B * (C + 1) * 4;
    s.chan = o;
    o += (size_t)max_ch * 4;
    o = (o + 15) & ~(size_t)15;  // 16-byte copies of the list blocks
    // The list blocks are read only while the channel list is built, before
    // the producer's first copy into the ring's last slot: they share that
    // slot when they fit in it.
    const size_t pf = (size_t)kS2Prefetch * kCB * 4;
    if (nstage >= 2 && pf <= (size_t)3 * d * 2) {
        s.chanpf = (size_t)(nstage - 1) * 3 * d * 2;
    } else {
        s.chanpf = o;
        o += pf;
    }
    s.total = (o + 127) & ~(size_t)127;
    return s;
}

namespace {

__device__ __forceinline__ uint4 lds128(const void *p) {
    return *reinterpret_cast<const uint4 *>(p);
}

// acc.x += w.lo * x.lo, acc.y += w.hi * x.hi for a word of two bf16 weights
// and two bf16 inputs: the products are exact in fp32 (8-bit significands),
// so this equals an fp32 FMA of the widened values, without widening them
__device__ __forceinline__ void fma_bf16_pair(float2 &acc, uint32_t w, uint32_t x) {
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\tmov.b32 {wl, wh}, %2;\n\tmov.b32 {xl, xh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, wl, xl, %0;\n\tfma.rn.f32.bf16 %1, wh, xh, %1;\n\t}"
        : "+f"(acc.x), "+f"(acc.y)
        : "r"(w), "r"(x));
}

__device__ __forceinline__ void bf16x8_to_f2(const uint4 &w, float2 (&o)[4]) {
    const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) o[q] = make_float2(bf16lo(a[q]), bf16hi(a[q]));
}

template <int B, int NCHD>
__global__ void __launch_bounds__(s2_threads(B), 1) k_stage2(const Stage2Args a) {
    constexpr int NDOWN = s2_ndown(B);
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int d = a.d, C = a.C, NST = a.nstage;
    const S2Smem L = s2_smem(d, B, NST, C, a.max_ch);
    uint16_t *stages = reinterpret_cast<uint16_t *>(smem + L.stages);
    uint16_t *xh = reinterpret_cast<uint16_t *>(smem + L.xs);  // x, bf16 [B][d]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.full);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + L.empty);
    uint64_t *sready = reinterpret_cast<uint64_t *>(smem + L.sready);
    uint32_t *meta = reinterpret_cast<uint32_t *>(smem + L.meta);
    float *svals = reinterpret_cast<float *>(smem + L.svals);  // [NST][B]
    int *uscan = reinterpret_cast<int *>(smem + L.uscan);      // [C+1]
    int *tscan = reinterpret_cast<int *>(smem + L.tscan);      // [B][C+1]
    uint32_t *chan = reinterpret_cast<uint32_t *>(smem + L.chan);  // [max_ch]
    uint32_t *chanpf = reinterpret_cast<uint32_t *>(smem + L.chanpf);  // [kS2Prefetch][kCB]
    const int nch16 = d / 8;  // 16-byte chunks per row

    if (tid == 0) {
        stamp_min(a.stamps, kS2Entry);
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + NDOWN);
            mbar_init(&sready[s], 1);
        }
        mbar_fence_init();
    }
    // x into shared memory as it is (bf16; the dot warps multiply bf16 pairs
    // into fp32 sums). Stage 1, the kernel this one may overlap, only
    // triggers this launch after its own griddepcontrol.wait, so x (written
    // before Stage 1 ran) is complete.
    for (int k = tid; k < B * nch16; k += s2_threads(B)) {
        const int t = k / nch16, ci = k % nch16;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < a.nb) v = *reinterpret_cast<const uint4 *>(a.x + (size_t)t * d + ci * 8);
        *reinterpret_cast<uint4 *>(xh + (size_t)t * d + ci * 8) = v;
    }
    // x and the barriers are in place before Stage 1 has finished
    __syncthreads();
    // Stage 1's lists are ready once it has completed. One round trip brings
    // the per-block counts and the list blocks this CTA most likely owns
    // (those around block g * C / G).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (tid == 0) {
        stamp_min(a.stamps, kS2Go);
        stamp_max(a.stamps, kS2GoMax);
    }
    asm volatile("griddepcontrol.launch_dependents;");
    // (G is one CTA per SM, so every product below fits in 32 bits)
    const int G = gridDim.x, g = blockIdx.x;
    const int npf = C < kS2Prefetch ? C : kS2Prefetch;
    int cpf = g * C / G - 1;
    cpf = cpf < 0 ? 0 : (cpf > C - npf ? C - npf : cpf);
    // per-token counts only when per-token lists or counts are requested
    const bool tok = a.idx_s != nullptr || a.count_s != nullptr;
    int n_ch;
    if (!tok && C <= 32 * 4) {
        // Every warp reads the union counts itself (lane l owns blocks 4 l ..
        // 4 l + 3) and derives this CTA's share [U g / G, U (g + 1) / G); the
        // producer warp also takes the likely list blocks in the same round
        // trip, scans the counts into shared memory and builds its channel
        // list, so its first copies go out with no CTA-wide barrier.
        const bool prod = wid == kNDot + NDOWN;
        int cnt[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) cnt[k] = lane * 4 + k < C ? a.ucount[lane * 4 + k] : 0;
        uint4 pf[kS2Prefetch * kCB / 4 / 32];
        if (prod) {
#pragma unroll
            for (int q = 0; q < kS2Prefetch * kCB / 4 / 32; ++q) {
                const int e = (q * 32 + lane) * 4;  // first of 4 list entries
                pf[q] = e < npf * kCB
                            ? *reinterpret_cast<const uint4 *>(a.ulist + (size_t)cpf * kCB + e)
                            : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        const int loc = cnt[0] + cnt[1] + cnt[2] + cnt[3];
        int inc = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        const unsigned U = (unsigned)__shfl_sync(0xffffffffu, inc, 31);
        const int p0 = (int)(U * g / G);
        n_ch = (int)(U * (g + 1) / G) - p0;
        if (prod) {
            int run = inc - loc;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (lane * 4 + k < C) uscan[lane * 4 + k] = run;
                run += cnt[k];
            }
            if (lane == 31) uscan[C] = inc;
#pragma unroll
            for (int q = 0; q < kS2Prefetch * kCB / 4 / 32; ++q) {
                const int e = (q * 32 + lane) * 4;
                if (e < npf * kCB) *reinterpret_cast<uint4 *>(chanpf + e) = pf[q];
            }
            __syncwarp();
            for (int n = lane; n < n_ch; n += 32) {
                const int pp = p0 + n;
                int lo = 0, hi = C - 1;  // block cb with uscan[cb] <= pp < uscan[cb + 1]
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (uscan[mid] <= pp) lo = mid; else hi = mid - 1;
                }
                const int off = pp - uscan[lo];
                chan[n] = (lo >= cpf && lo < cpf + npf) ? chanpf[(lo - cpf) * kCB + off]
                                                        : a.ulist[(size_t)lo * kCB + off];
            }
            __syncwarp();
            if (lane == 0) stamp_max(a.stamps, kS2List);
        }
    } else {
        constexpr int NT = s2_threads(B);
        // Warp 0 takes the union counts into registers (4 per lane covers
        // C <= 128 column blocks; more go through shared memory), every thread a
        // share of the likely list blocks and, when asked for, of the per-token
        // counts: all loads of this round trip are issued before any is used.
        constexpr int PER = 4;
        const bool creg = C <= 32 * PER;
        int cnt[PER];
#pragma unroll
        for (int k = 0; k < PER; ++k) cnt[k] = 0;
        if (wid == 0 && creg) {
#pragma unroll
            for (int k = 0; k < PER; ++k)
                if (lane * PER + k < C) cnt[k] = a.ucount[lane * PER + k];
        }
        {
            const int nuc = creg ? 0 : C;          // union counts via shared memory
            const int ntc = tok ? C * B : 0;       // per-token counts
            const int total = nuc + ntc + npf * kCB;
            for (int base = tid; base < total; base += 4 * NT) {
                uint32_t v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int k = base + q * NT;
                    v[q] = 0;
                    if (k < nuc) v[q] = (uint32_t)a.ucount[k];
                    else if (k < nuc + ntc)  // one token: the union's counts are its own
                        v[q] = (uint32_t)(B == 1 ? a.ucount[k - nuc] : a.tcount[k - nuc]);
                    else if (k < total) v[q] = a.ulist[(size_t)cpf * kCB + (k - nuc - ntc)];
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int k = base + q * NT;
                    if (k < nuc) {
                        uscan[k] = (int)v[q];
                    } else if (k < nuc + ntc) {
                        const int c = (k - nuc) / B, t = (k - nuc) % B;
                        tscan[t * (C + 1) + c] = (int)v[q];
                    } else if (k < total) {
                        chanpf[k - nuc - ntc] = v[q];
                    }
                }
            }
        }
        __syncthreads();
        // Exclusive scans of the per-block counts: warp 0 the union counts (in
        // registers), warp 1 + t those of token t (in place). A lane owns
        // contiguous counts, so one shuffle scan suffices.
        if (wid == 0 && creg) {
            int loc = 0;
#pragma unroll
            for (int k = 0; k < PER; ++k) loc += cnt[k];
            int inc = loc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += n;
            }
            int run = inc - loc;
#pragma unroll
            for (int k = 0; k < PER; ++k) {
                if (lane * PER + k < C) uscan[lane * PER + k] = run;
                run += cnt[k];
            }
            if (lane == 31) uscan[C] = inc;
        } else if (wid == 0 || (tok && wid <= B)) {
            int *dst = (wid == 0) ? uscan : tscan + (wid - 1) * (C + 1);
            const int per = (C + 31) / 32;
            const int c0 = lane * per;
            int loc = 0;
            for (int k = 0; k < per; ++k)
                if (c0 + k < C) loc += dst[c0 + k];
            int inc = loc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += n;
            }
            int run = inc - loc;
            for (int k = 0; k < per; ++k)
                if (c0 + k < C) {
                    const int v = dst[c0 + k];
                    dst[c0 + k] = run;
                    run += v;
                }
            if (lane == 31) dst[C] = inc;
        }
        // warp 0: this CTA's share of the ascending kept-channel list
        if (wid == 0) {
            __syncwarp();
            const unsigned U = (unsigned)uscan[C];  // <= 2^18 kept channels
            const int p0 = (int)(U * g / G), p1 = (int)(U * (g + 1) / G);
            for (int n = lane; n < p1 - p0; n += 32) {
                const int p = p0 + n;
                int lo = 0, hi = C - 1;  // block cb with uscan[cb] <= p < uscan[cb + 1]
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (uscan[mid] <= p) lo = mid; else hi = mid - 1;
                }
                const int off = p - uscan[lo];
                chan[n] = (lo >= cpf && lo < cpf + npf) ? chanpf[(lo - cpf) * kCB + off]
                                                        : a.ulist[(size_t)lo * kCB + off];
            }
        }
        __syncthreads();
        if (tid == 0) stamp_max(a.stamps, kS2List);
        const unsigned U = (unsigned)uscan[C];
        n_ch = (int)(U * (g + 1) / G) - (int)(U * g / G);
    }

    if (wid == kNDot + NDOWN) {
        // ---------------- producer ----------------
        if (lane != 0) return;
        const uint32_t row_bytes = (uint32_t)d * 2;
        const uint64_t pol = l2_evict_first();  // each weight row is read once per pass
        int issued = 0;
        for (int n = 0; n < n_ch; ++n) {
            const uint32_t e = chan[n];
            const int s = n % NST, k = n / NST;
            if (k > 0 && !mbar_wait(&empty[s], (k - 1) & 1, a.spin_limit)) {
                atomicOr(a.status, kStTimeoutEmpty);
                break;
            }
            meta[s] = e;
            issued = n + 1;
            if (a.debug_skip == n && g == 0) continue;  // test hook: stage never filled
            const size_t j = e & 0xFFFFFFu;
            uint16_t *dst = stages + (size_t)s * 3 * d;
            mbar_arrive_expect_tx(&full[s], 3 * row_bytes);
            bulk_g2s_hint(dst, a.w_up + j * d, row_bytes, &full[s], pol);
            bulk_g2s_hint(dst + d, a.w_gate + j * d, row_bytes, &full[s], pol);
            bulk_g2s_hint(dst + 2 * d, a.w_down + j * d, row_bytes, &full[s], pol);
        }
        // never leave the CTA with copies in flight
        const int first = issued > NST ? issued - NST : 0;
        for (int n = first; n < issued; ++n) {
            if (a.debug_skip == n && g == 0) continue;
            if (!mbar_wait(&full[n % NST], (n / NST) & 1, a.spin_limit)) {
                atomicOr(a.status, kStTimeoutDrain);
                break;
            }
        }
        return;
    }

    if (wid < kNDot) {
        // ---------------- dot warps: u_j, g_j, s_j ----------------
        // Slot s always belongs to dot warp s % kNDot, so a warp waits on each
        // of its slots' phases in order (a parity wait is only meaningful once
        // the slot's previous phase has been observed by the same waiter).
        for (int n = 0; n < n_ch; ++n) {
            const int s = n % NST, k = n / NST;
            if (s % kNDot != wid) continue;
            // the decision to give up is warp-uniform (lanes share later shuffles)
            if (!__all_sync(0xffffffffu, mbar_wait(&full[s], k & 1, a.spin_limit))) {
                if (lane == 0) atomicOr(a.status, kStTimeoutFull);
                break;
            }
            if (n == 0 && lane == 0) {
                stamp_min(a.stamps, kS2First);
                stamp_max(a.stamps, kS2FirstMax);
            }
            const uint32_t bits = (B == 1) ? 1u : (meta[s] >> 24);
            const uint16_t *up = stages + (size_t)s * 3 * d;
            const uint16_t *gt = up + d;
            float2 u2[B], g2[B];
#pragma unroll
            for (int t = 0; t < B; ++t) u2[t] = g2[t] = make_float2(0.f, 0.f);
            for (int ci = lane; ci < nch16; ci += 32) {
                const uint4 wu = lds128(up + ci * 8), wg = lds128(gt + ci * 8);
#pragma unroll
                for (int t = 0; t < B; ++t) {
                    if (B > 1 && !((bits >> t) & 1u)) continue;
                    const uint4 xq = lds128(xh + (size_t)t * d + ci * 8);
                    fma_bf16_pair(u2[t], wu.x, xq.x);
                    fma_bf16_pair(u2[t], wu.y, xq.y);
                    fma_bf16_pair(u2[t], wu.z, xq.z);
                    fma_bf16_pair(u2[t], wu.w, xq.w);
                    fma_bf16_pair(g2[t], wg.x, xq.x);
                    fma_bf16_pair(g2[t], wg.y, xq.y);
                    fma_bf16_pair(g2[t], wg.z, xq.z);
                    fma_bf16_pair(g2[t], wg.w, xq.w);
                }
            }
            float sv[B];
#pragma unroll
            for (int t = 0; t < B; ++t) {
                float u = u2[t].x + u2[t].y, gg = g2[t].x + g2[t].y;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    u += __shfl_xor_sync(0xffffffffu, u, o);
                    gg += __shfl_xor_sync(0xffffffffu, gg, o);
                }
                sv[t] = ((bits >> t) & 1u) ? u * gate_act(gg, a.act) : 0.f;
            }
            __syncwarp();
            if (lane == 0) {
#pragma unroll
                for (int t = 0; t < B; ++t) svals[s * B + t] = sv[t];
                mbar_arrive(&sready[s]);
                mbar_arrive(&empty[s]);  // done with the up/gate rows
            }
        }
        // per-token ascending kept-channel lists (blocks c = g, g + G, ...)
        if (a.idx_s) {
            for (int c = g; c < C; c += G) {
                for (int t = 0; t < a.nb; ++t) {
                    const int nk = B == 1 ? a.ucount[c] : a.tcount[c * B + t];
                    const int base = tscan[t * (C + 1) + c];
                    for (int k = tid; k < nk; k += kNDot * 32)
                        a.idx_s[(size_t)t * a.f + base + k] =
                            B == 1 ? (int32_t)(a.ulist[(size_t)c * kCB + k] & 0xFFFFFFu)
                                   : a.tlist[(size_t)t * a.f + c * kCB + k];
                }
            }
        }
        if (g == 0 && a.count_s && tid < a.nb) a.count_s[tid] = tscan[tid * (C + 1) + C];
        return;
    }

    // ---------------- down warps: y slice += s_j * W_down[j, slice] ----------
    const int dt = tid - kNDot * 32;
    float2 acc[B][NCHD][4];
#pragma unroll
    for (int t = 0; t < B; ++t)
#pragma unroll
        for (int m = 0; m < NCHD; ++m)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[t][m][q] = make_float2(0.f, 0.f);

    for (int n = 0; n < n_ch; ++n) {
        const int s = n % NST, ph = (n / NST) & 1;
        const bool ok = mbar_wait(&full[s], ph, a.spin_limit) &&
                        mbar_wait(&sready[s], ph, a.spin_limit);
        if (!__all_sync(0xffffffffu, ok)) {  // warp-uniform decision
            if (lane == 0) atomicOr(a.status, kStTimeoutRed);
            break;
        }
        const uint32_t bits = (B == 1) ? 1u : (meta[s] >> 24);
        float sv[B];
#pragma unroll
        for (int t = 0; t < B; ++t) sv[t] = svals[s * B + t];
        const uint16_t *dn = stages + (size_t)s * 3 * d + 2 * d;
#pragma unroll
        for (int m = 0; m < NCHD; ++m) {
            const int ci = dt + m * NDOWN * 32;
            if (ci < nch16) {
                float2 w[4];
                bf16x8_to_f2(lds128(dn + ci * 8), w);
#pragma unroll
                for (int t = 0; t < B; ++t) {
                    if (B > 1 && !((bits >> t) & 1u)) continue;
                    const float2 ss = make_float2(sv[t], sv[t]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[t][m][q] = __ffma2_rn(ss, w[q], acc[t][m][q]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (lane == 0) stamp_max(a.stamps, kS2Stream);

    if (n_ch == 0) return;
    // The CTA's partial y goes to global memory as one bulk reduction (the
    // copy engine adds a shared-memory copy of it into y), not as one 16-byte
    // atomic per thread and chunk. Every down warp is past its last stage, and
    // the dot warps and the producer are done with theirs, so the ring is free
    // for that copy once all down warps are here.
    named_bar_sync(1, NDOWN * 32);
    float *ys = reinterpret_cast<float *>(stages);  // [nb][d]
#pragma unroll
    for (int t = 0; t < B; ++t) {
        if (t >= a.nb) break;
#pragma unroll
        for (int m = 0; m < NCHD; ++m) {
            const int ci = dt + m * NDOWN * 32;
            if (ci < nch16) {
                float4 *dst = reinterpret_cast<float4 *>(ys + (size_t)t * d + ci * 8);
                dst[0] = make_float4(acc[t][m][0].x, acc[t][m][0].y, acc[t][m][1].x, acc[t][m][1].y);
                dst[1] = make_float4(acc[t][m][2].x, acc[t][m][2].y, acc[t][m][3].x, acc[t][m][3].y);
            }
        }
    }
    fence_proxy_async_smem();  // the copy engine reads what these threads wrote
    named_bar_sync(1, NDOWN * 32);
    if (dt == 0) {
        bulk_reduce_add_f32(a.y, ys, (uint32_t)(a.nb * d * 4));
        stamp_max(a.stamps, kS2End);
    }
}

template <int B, int NCHD>
cudaError_t launch2(const Stage2Args &a, int grid, size_t smem, cudaStream_t s) {
    auto k = k_stage2<B, NCHD>;
    cudaError_t e = set_max_dynamic_smem((const void *)k, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3(grid), dim3(s2_threads(B)), smem, s, a);
}

}  // namespace

// chunks of 8 columns each down thread owns (a power of two)
int stage2_nchd(int d_model, int B) {
    const int per = (d_model / 8 + s2_ndown(B) * 32 - 1) / (s2_ndown(B) * 32);
    int p = 1;
    while (p < per) p <<= 1;
    return p;
}

cudaError_t launch_stage2(int B, int nchd, const Stage2Args &a, int grid, size_t smem,
                          cudaStream_t s) {
#define PROX_S2(BB, NN) \
    if (B == BB && nchd == NN) return launch2<BB, NN>(a, grid, smem, s);
    PROX_S2(1, 1) PROX_S2(1, 2) PROX_S2(1, 4)
    PROX_S2(2, 1) PROX_S2(2, 2) PROX_S2(2, 4)
    PROX_S2(4, 1) PROX_S2(4, 2)
    PROX_S2(8, 1)
#undef PROX_S2
    return cudaErrorInvalidValue;
}

size_t stage2_smem_bytes(int d_model, int B, int nstage, int C, int max_ch) {
    return s2_smem(d_model, B, nstage, C, max_ch).total;
}

}  // namespace prox
