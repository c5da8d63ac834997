// Stage 2 of the Prox sparse SwiGLU FFN on sm_100a: exact output-sparse
// up/gate over the kept channels, SiLU-mul, and the input-sparse down
// projection over the same channels (Prox deep-dive blog, section "Stage 2";
// Pi_out / Pi_in of the translated arXiv page, section 2.2; the weighted-sum
// view y = sum_j s_j W_down[j, :] of the blog's first section).
//
// One persistent CTA per SM takes an equal share of the kept channels (the
// union over the pass's tokens, in ascending order). W_up and W_gate are
// stored channel-major and W_down row-major, so a kept channel j is three
// contiguous d_model-long bf16 rows. A producer lane moves them with 1-D bulk
// copies (TMA) into a ring of shared-memory stages guarded by mbarriers;
// 16 consumer warps each own a 1/16 slice of the d_model columns: they form
// partial dot products x . W_up[j] and x . W_gate[j] on their slice, exchange
// them through shared memory (an mbarrier, not a hardware barrier, so every
// wait is bounded), compute s_j = u_j * SiLU(g_j) in fp32 and accumulate
// s_j * W_down[j, slice] into registers. At the end each CTA adds its partial
// y to global memory with 16-byte vector reductions.
#include "prox_internal.cuh"

#include <cuda_runtime.h>
#include <cstdint>

namespace prox {

// shared-memory carve-up, shared by the kernel and the host plan
struct S2Smem {
    size_t stages, xs, full, empty, redbar, meta, red, uscan, tscan, chan, total;
};

__host__ __device__ inline S2Smem s2_smem(int d, int B, int nstage, int C, int max_ch) {
    S2Smem s;
    size_t o = 0;
    s.stages = o;
    o += (size_t)nstage * 3 * d * 2;
    s.xs = o;
    o += (size_t)B * d * 2;
    o = (o + 15) & ~(size_t)15;
    s.full = o;
    o += (size_t)nstage * 8;
    s.empty = o;
    o += (size_t)nstage * 8;
    s.redbar = o;
    o += 2 * 8;
    s.meta = o;
    o += (size_t)nstage * 4;
    o = (o + 15) & ~(size_t)15;
    s.red = o;
    o += (size_t)2 * kNCW * 2 * B * 4;
    s.uscan = o;
    o += (size_t)(C + 1) * 4;
    s.tscan = o;
    o += (size_t)B * (C + 1) * 4;
    s.chan = o;
    o += (size_t)max_ch * 4;
    s.total = (o + 127) & ~(size_t)127;
    return s;
}

namespace {

__device__ __forceinline__ uint4 lds128(const void *p) {
    return *reinterpret_cast<const uint4 *>(p);
}

// acc += x . w over 8 bf16 pairs
__device__ __forceinline__ float dot8(const uint4 &x, const uint4 &w, float acc) {
    const uint32_t xa[4] = {x.x, x.y, x.z, x.w};
    const uint32_t wa[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        acc = fmaf(bf16lo(xa[q]), bf16lo(wa[q]), acc);
        acc = fmaf(bf16hi(xa[q]), bf16hi(wa[q]), acc);
    }
    return acc;
}

template <int B, int NCH>
__global__ void __launch_bounds__(kS2Threads, 1) k_stage2(const Stage2Args a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int d = a.d, C = a.C, NST = a.nstage;
    const S2Smem L = s2_smem(d, B, NST, C, a.max_ch);
    uint16_t *stages = reinterpret_cast<uint16_t *>(smem + L.stages);
    uint16_t *xsm = reinterpret_cast<uint16_t *>(smem + L.xs);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.full);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + L.empty);
    uint64_t *redbar = reinterpret_cast<uint64_t *>(smem + L.redbar);
    uint32_t *meta = reinterpret_cast<uint32_t *>(smem + L.meta);
    float *red = reinterpret_cast<float *>(smem + L.red);  // [2][kNCW][B][2]
    int *uscan = reinterpret_cast<int *>(smem + L.uscan);  // [C+1]
    int *tscan = reinterpret_cast<int *>(smem + L.tscan);  // [B][C+1]
    uint32_t *chan = reinterpret_cast<uint32_t *>(smem + L.chan);  // [max_ch]
    const int nch16 = d / 8;  // 16-byte chunks per row

    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kNCW);
        }
        mbar_init(&redbar[0], kNCW);
        mbar_init(&redbar[1], kNCW);
        mbar_fence_init();
    }
    // x (bf16) into shared memory; tokens beyond nb are zero. Stage 1, the
    // kernel this one may overlap, only triggers this launch after its own
    // griddepcontrol.wait, so x (written before Stage 1 ran) is complete.
    for (int k = tid; k < B * nch16; k += kS2Threads) {
        const int t = k / nch16, ci = k % nch16;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < a.nb) v = *reinterpret_cast<const uint4 *>(a.x + (size_t)t * d + ci * 8);
        *reinterpret_cast<uint4 *>(xsm + (size_t)t * d + ci * 8) = v;
    }
    // Stage 1's lists are ready once it has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int k = tid; k < C * (B + 1); k += kS2Threads) {
        if (k < C) {
            uscan[k] = a.ucount[k];
        } else {
            const int c = (k - C) / B, t = (k - C) % B;
            tscan[t * (C + 1) + c] = a.tcount[c * B + t];
        }
    }
    __syncthreads();
    // exclusive scans of the per-block counts, in place (warp 0)
    if (wid == 0) {
        for (int t = -1; t < B; ++t) {
            int carry = 0;
            int *dst = (t < 0) ? uscan : tscan + t * (C + 1);
            for (int c0 = 0; c0 < C; c0 += 32) {
                const int c = c0 + lane;
                const int v = (c < C) ? dst[c] : 0;
                int inc = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int n = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += n;
                }
                if (c < C) dst[c] = carry + inc - v;
                carry += __shfl_sync(0xffffffffu, inc, 31);
            }
            if (lane == 0) dst[C] = carry;
        }
    }
    __syncthreads();

    const long long U = uscan[C];
    const int G = gridDim.x, g = blockIdx.x;
    const int p0 = (int)(U * g / G), p1 = (int)(U * (g + 1) / G);
    const int n_ch = p1 - p0;

    // this CTA's share of the ascending kept-channel list, into shared memory
    for (int n = tid; n < n_ch; n += kS2Threads) {
        const int p = p0 + n;
        int lo = 0, hi = C - 1;  // block cb with uscan[cb] <= p < uscan[cb + 1]
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (uscan[mid] <= p) lo = mid; else hi = mid - 1;
        }
        chan[n] = a.ulist[(size_t)lo * kCB + (p - uscan[lo])];
    }
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;");

    if (wid == kNCW) {
        // ---------------- producer ----------------
        if (lane != 0) return;
        const uint32_t row_bytes = (uint32_t)d * 2;
        int issued = 0;
        bool ok = true;
        for (int n = 0; n < n_ch; ++n) {
            const uint32_t e = chan[n];
            const int s = n % NST, k = n / NST;
            if (k > 0 && !mbar_wait(&empty[s], (k - 1) & 1, a.spin_limit)) {
                atomicOr(a.status, kStTimeoutEmpty);
                ok = false;
                break;
            }
            meta[s] = e;
            issued = n + 1;
            if (a.debug_skip == n && g == 0) continue;  // test hook: stage never filled
            const size_t j = e & 0xFFFFFFu;
            uint16_t *dst = stages + (size_t)s * 3 * d;
            mbar_arrive_expect_tx(&full[s], 3 * row_bytes);
            bulk_g2s(dst, a.w_up + j * d, row_bytes, &full[s]);
            bulk_g2s(dst + d, a.w_gate + j * d, row_bytes, &full[s]);
            bulk_g2s(dst + 2 * d, a.w_down + j * d, row_bytes, &full[s]);
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
        (void)ok;
        return;
    }

    // ---------------- consumers ----------------
    float yacc[B][NCH][8];
#pragma unroll
    for (int t = 0; t < B; ++t)
#pragma unroll
        for (int q = 0; q < NCH; ++q)
#pragma unroll
            for (int k = 0; k < 8; ++k) yacc[t][q][k] = 0.f;

    for (int n = 0; n < n_ch; ++n) {
        const int s = n % NST, k = n / NST;
        if (!mbar_wait(&full[s], k & 1, a.spin_limit)) {
            if (lane == 0) atomicOr(a.status, kStTimeoutFull);
            break;
        }
        const uint32_t bits = meta[s] >> 24;
        const uint16_t *up = stages + (size_t)s * 3 * d;
        const uint16_t *gt = up + d;
        const uint16_t *dn = up + 2 * d;

        float pu[B], pg[B];
#pragma unroll
        for (int t = 0; t < B; ++t) pu[t] = pg[t] = 0.f;
#pragma unroll
        for (int q = 0; q < NCH; ++q) {
            const int ci = tid + q * kNCW * 32;
            if (ci < nch16) {
                const uint4 wu = lds128(up + ci * 8);
                const uint4 wg = lds128(gt + ci * 8);
#pragma unroll
                for (int t = 0; t < B; ++t) {
                    if (!((bits >> t) & 1u)) continue;
                    const uint4 xv = lds128(xsm + (size_t)t * d + ci * 8);
                    pu[t] = dot8(xv, wu, pu[t]);
                    pg[t] = dot8(xv, wg, pg[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < B; ++t) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                pu[t] += __shfl_xor_sync(0xffffffffu, pu[t], o);
                pg[t] += __shfl_xor_sync(0xffffffffu, pg[t], o);
            }
        }
        float *rb = red + (size_t)(n & 1) * kNCW * B * 2;
        if (lane == 0) {
#pragma unroll
            for (int t = 0; t < B; ++t) {
                rb[(wid * B + t) * 2 + 0] = pu[t];
                rb[(wid * B + t) * 2 + 1] = pg[t];
            }
            mbar_arrive(&redbar[n & 1]);
        }
        if (!mbar_wait(&redbar[n & 1], (n >> 1) & 1, a.spin_limit)) {
            if (lane == 0) atomicOr(a.status, kStTimeoutRed);
            break;
        }
        float sv[B];
#pragma unroll
        for (int t = 0; t < B; ++t) {
            float u = 0.f, gg = 0.f;
            if ((bits >> t) & 1u) {
#pragma unroll
                for (int w = 0; w < kNCW; ++w) {
                    u += rb[(w * B + t) * 2 + 0];
                    gg += rb[(w * B + t) * 2 + 1];
                }
            }
            sv[t] = ((bits >> t) & 1u) ? u * (gg / (1.f + expf(-gg))) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < NCH; ++q) {
            const int ci = tid + q * kNCW * 32;
            if (ci < nch16) {
                const uint4 wd = lds128(dn + ci * 8);
                const uint32_t wa[4] = {wd.x, wd.y, wd.z, wd.w};
#pragma unroll
                for (int t = 0; t < B; ++t) {
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        yacc[t][q][2 * h] = fmaf(sv[t], bf16lo(wa[h]), yacc[t][q][2 * h]);
                        yacc[t][q][2 * h + 1] = fmaf(sv[t], bf16hi(wa[h]), yacc[t][q][2 * h + 1]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }

    // per-token ascending kept-channel lists (blocks c = g, g + G, ...)
    if (a.idx_s) {
        for (int c = g; c < C; c += G) {
            for (int t = 0; t < a.nb; ++t) {
                const int n = a.tcount[c * B + t];
                const int base = tscan[t * (C + 1) + c];
                for (int k = tid; k < n; k += kNCW * 32)
                    a.idx_s[(size_t)t * a.f + base + k] = a.tlist[(size_t)t * a.f + c * kCB + k];
            }
        }
    }
    if (g == 0 && a.count_s && tid < a.nb) a.count_s[tid] = tscan[tid * (C + 1) + C];

    if (n_ch == 0) return;
#pragma unroll
    for (int t = 0; t < B; ++t) {
        if (t >= a.nb) break;
#pragma unroll
        for (int q = 0; q < NCH; ++q) {
            const int ci = tid + q * kNCW * 32;
            if (ci < nch16) {
                float *dst = a.y + (size_t)t * d + ci * 8;
                red_add_v4(dst, yacc[t][q][0], yacc[t][q][1], yacc[t][q][2], yacc[t][q][3]);
                red_add_v4(dst + 4, yacc[t][q][4], yacc[t][q][5], yacc[t][q][6], yacc[t][q][7]);
            }
        }
    }
}

template <int B, int NCH>
cudaError_t launch2(const Stage2Args &a, int grid, size_t smem, cudaStream_t s) {
    auto k = k_stage2<B, NCH>;
    static size_t configured = 0;  // dynamic smem limit already set for this kernel
    if (smem > configured) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        configured = smem;
    }
    return launch_pdl(k, dim3(grid), dim3(kS2Threads), smem, s, a);
}

}  // namespace

cudaError_t launch_stage2(int B, int nchunk, const Stage2Args &a, int grid, size_t smem,
                          cudaStream_t s) {
#define PROX_S2(BB, NN) \
    if (B == BB && nchunk == NN) return launch2<BB, NN>(a, grid, smem, s);
    PROX_S2(1, 1) PROX_S2(1, 2) PROX_S2(1, 4) PROX_S2(1, 8)
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
