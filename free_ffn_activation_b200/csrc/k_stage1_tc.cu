// Stage 1 of the Prox sparse SwiGLU FFN on the tensor cores, for passes of
// 1, 2 or 4 tokens with the INT4 proxy (Prox deep-dive blog, section
// "Stage 1"; input-sparse projection Pi_in of the translated arXiv page,
// section 2.2): input masks, the proxy products u~ = Pi_in(x, W~_up, m_x)
// and g~ = Pi_in(x, W~_gate, m_x), s~ = u~ * SiLU(g~), the channel masks and
// the ascending kept-channel lists Stage 2 reads.
//
// Arithmetic. The proxy product of channel j is sum_i q_ij x_i scale_i over
// the kept rows i. x_i * scale_i (per matrix and token) becomes a 27-bit
// fixed-point integer v_i = round(x_i scale_i 2^F), F one exponent per
// (matrix, token) shared by the whole grid, split into four signed 8-bit
// digits v = d0 + 2^7 d1 + 2^14 d2 + 2^21 d3. The codes (stored offset
// binary, n = q + 8) are the A operand of tcgen05.mma kind::i8 as unsigned
// bytes, the digits the B operand (4 digit rows per token, N = 16), and the
// int32 accumulation in tensor memory is exact. Per channel the CTA's
// partial sum_i q_ij v_i is then an exact int64, and the partials of the
// CTAs that share a column block add up exactly (in any order) in int64
// global accumulators: the result equals sum_i q_ij round(x_i scale_i 2^F)
// times 2^-F whatever the split.
//
// Decode. A 32-bit word of the proxy holds 8 codes, the even channels in the
// low nibbles. w & 0x0F0F0F0F gives the 4 even channels as bytes and
// w & 0xF0F0F0F0 the 4 odd ones times 16: two ANDs per 8 codes. A 16-byte
// chunk of one row (32 channels) thus becomes 16 bytes of even channels and
// 16 bytes of odd channels x 16, stored as two 16-byte pieces of the A tile:
// the M order of the tile is permuted within each group of 32 channels and
// the odd half carries a factor 16, both undone in the epilogue (the factor
// exactly: its int32 sums are multiples of 16).
//
// Work split. Column block c (256 channels of both proxies) is covered by
// n_r CTAs (no cluster), CTA r taking the r-th contiguous range of the kept
// rows (ranks over the union of the pass's tokens). Roles of the 17 warps:
//   warps 0..15  each thread owns one 16-byte piece of every K step (32 kept
//                rows x 2 proxies x 128 bytes): it loads the pieces of the
//                next 8 K steps into registers (L2 evict-first), decodes the
//                current one into the swizzled A tiles of a ring of K steps,
//                makes them visible to the tensor core (fence.proxy.async)
//                and its warp arrives on "A full";
//   warp 16      issues the 4 MMAs of each K step (2 proxies x 2 M tiles of
//                128 channels) and frees ring slots with tcgen05.commit;
//   warps 0..15  then read the accumulators (one (proxy, M tile) and lane
//                quadrant per warp) and add the CTA's partials to the int64
//                accumulators of the block with red.global.add.
// A 128-byte granule is too small a copy for the TMA engine to stream at
// HBM rate; 16-byte loads from all threads with 8 steps in flight are not.
// The last CTA of a block to arrive (a counter per block) turns the exact
// sums into fp32 u~, g~, forms s~, the masks and the lists. The host clears
// the accumulators and counters on the stream before each pass. Every wait is
// bounded; on a timeout the CTA records status bit 4 and skips ahead, and
// tensor memory is freed before exit.
#include "prox_internal.cuh"
#include "umma.cuh"

#include <cuda_runtime.h>
#include <cstdint>

namespace prox {

namespace {

constexpr int kDecW = 16;           // warps 0..15: load + decode, then epilogue
constexpr int kMmaW = 16;           // warp 16: MMA issue
constexpr int kT = (kDecW + 1) * 32;
constexpr int kKS = 32;             // proxy rows per K step (K of one kind::i8 MMA)
constexpr int kN = 16;              // digit rows: 4 per token, up to 4 tokens
constexpr int kPre = 8;             // K steps each thread has in flight
constexpr uint32_t kATile = kKS * 128;           // one (proxy, M tile) A tile of a K step
constexpr uint32_t kAStep = 4 * kATile;          // the 4 A tiles of a K step
constexpr int kASlots = 6;
// kind::i8: s32 D, u8 A (MN-major), s8 B (K-major), N = 16, M = 128
constexpr uint32_t kIdesc = (2u << 4) | (0u << 7) | (1u << 10) | (1u << 15) |
                            ((uint32_t)(kN >> 3) << 17) | (8u << 24);

struct TcSmem {
    uint32_t a, dig, rowidx, bars, total;
};
// offsets from a 1024-byte aligned base; unit_cap = most kept rows of a CTA
__host__ __device__ inline TcSmem tc_smem(int unit_cap) {
    const int nks = (unit_cap + kKS - 1) / kKS;
    const int nkb = (nks * kKS + 127) / 128;   // 128-row digit blocks
    TcSmem s;
    uint32_t o = 0;
    s.a = o;
    o += kASlots * kAStep;
    s.dig = o;                                 // [2 proxies][nkb][2 atoms][1024]
    o += 2u * nkb * 2048u;
    s.rowidx = o;
    o += (uint32_t)nks * kKS * 4;
    s.bars = o;
    o += (2 * kASlots + 2) * 8;
    s.total = o + 1024;                        // alignment slack of the dynamic base
    return s;
}

// global -> registers, 16 bytes, read-only path, under L2 policy pol
__device__ __forceinline__ uint4 ldg16(const void *src, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(src), "l"(pol));
    return v;
}

// byte offset, inside the digit region of one proxy, of digit row n (0..15)
// at proxy row (K) u: K-major, 128-byte swizzle, atoms of 8 rows x 128 K
__device__ __forceinline__ uint32_t dig_off(int u, int n) {
    return (uint32_t)(u >> 7) * 2048u + (uint32_t)(n >> 3) * 1024u + (uint32_t)(n & 7) * 128u +
           ((uint32_t)(((u & 127) >> 4) ^ (n & 7)) << 4) + (uint32_t)(u & 15);
}

// Bounded wait shared by the CTA: once any wait has given up, later ones
// return at once
__device__ __forceinline__ bool s1_wait(uint64_t *bar, uint32_t parity, const Stage1Args &a,
                                        volatile int *fail) {
    if (*fail) return false;
    if (mbar_wait(bar, parity, a.wait_us)) return true;
    *fail = 1;
    atomicOr(a.status, kStTimeoutRing);
    return false;
}

template <int B>
__global__ void __launch_bounds__(kT, 1) k_stage1_tc(const Stage1Args a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const uint32_t sbase = (smem_addr(smem_raw) + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (sbase - smem_addr(smem_raw));
    const TcSmem L = tc_smem(a.unit_cap);
    const int nr = a.n_r;
    const int c0 = blockIdx.x / nr;           // column block
    const int r = blockIdx.x % nr;            // row range of the block
    int *rowidx = reinterpret_cast<int *>(sm + L.rowidx);
    uint64_t *a_full = reinterpret_cast<uint64_t *>(sm + L.bars);
    uint64_t *a_empty = a_full + kASlots;
    uint64_t *done = a_empty + kASlots;
    __shared__ int s_warp[kT / 32];
    __shared__ float s_wmax[kT / 32][2 * kMaxB];
    __shared__ int s_F[2][4];
    __shared__ int s_S[2][4][4];
    __shared__ int s_cnt[kT / 32][kMaxB + 1];
    __shared__ uint32_t s_tmem;
    __shared__ int s_last;
    __shared__ volatile int s_fail;

    if (tid == 0) {
        stamp_min(a.stamps, kS1Entry);
        for (int s = 0; s < kASlots; ++s) {
            mbar_init(&a_full[s], kDecW);
            mbar_init(&a_empty[s], 1);
        }
        mbar_init(done, 1);
        mbar_fence_init();
        s_fail = 0;
    }
    if (tid < 2 * 4 * 4) (&s_S[0][0][0])[tid] = 0;
    if (wid == kMmaW) tmem_alloc(&s_tmem, 64);

    // The scales are layer weights: load this thread's 8 of each before the
    // previous kernel of the stream has finished.
    const int NC = a.d / 8;                   // 8-coordinate chunks (<= kT)
    const bool own = tid < NC;
    float4 su[2], sg[2];
    su[0] = su[1] = sg[0] = sg[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (own) {
        su[0] = *reinterpret_cast<const float4 *>(a.s_up + tid * 8);
        su[1] = *reinterpret_cast<const float4 *>(a.s_up + tid * 8 + 4);
        sg[0] = *reinterpret_cast<const float4 *>(a.s_gate + tid * 8);
        sg[1] = *reinterpret_cast<const float4 *>(a.s_gate + tid * 8 + 4);
    }

    // x, y and the workspace may belong to the previous kernel in the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    if (tid == 0) {
        stamp_min(a.stamps, kS1Go);
        stamp_max(a.stamps, kS1GoMax);
    }
    uint4 xv[B];
#pragma unroll
    for (int t = 0; t < B; ++t) {
        xv[t] = make_uint4(0u, 0u, 0u, 0u);
        if (own && t < a.nb) xv[t] = *reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.d + tid * 8);
    }
    // Stage 2 accumulates y with atomics: clear it (or start it from the
    // residual stream); clear the tensor-core Stage 2's atomics buffers
    if (a.y_zero) {
        float4 *y4 = reinterpret_cast<float4 *>(a.y_zero);
        const float4 *i4 = reinterpret_cast<const float4 *>(a.y_init);
        const int n4 = a.nb * a.d / 4;
        for (int k = blockIdx.x * kT + tid; k < n4; k += gridDim.x * kT)
            y4[k] = i4 ? i4[k] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (a.z_clear)
        for (int k = blockIdx.x * kT + tid; k < a.z_n16; k += gridDim.x * kT)
            a.z_clear[k] = make_uint4(0u, 0u, 0u, 0u);
    // digits of rows past the CTA's last and of absent tokens stay zero
    {
        const int nkb = ((a.unit_cap + kKS - 1) / kKS * kKS + 127) / 128;
        uint4 *dz = reinterpret_cast<uint4 *>(sm + L.dig);
        for (int k = tid; k < nkb * 2 * 2048 / 16; k += kT) dz[k] = make_uint4(0u, 0u, 0u, 0u);
    }

    // (1) keep bits per token, union bits, max |x_i scale_i| per (proxy, token)
    uint32_t kb[B], ub = 0;
    const float sus[8] = {su[0].x, su[0].y, su[0].z, su[0].w, su[1].x, su[1].y, su[1].z, su[1].w};
    const float sgs[8] = {sg[0].x, sg[0].y, sg[0].z, sg[0].w, sg[1].x, sg[1].y, sg[1].z, sg[1].w};
    float mx[2][B];
#pragma unroll
    for (int t = 0; t < B; ++t) {
        const uint32_t w4[4] = {xv[t].x, xv[t].y, xv[t].z, xv[t].w};
        uint32_t bits = 0;
        mx[0][t] = mx[1][t] = 0.f;
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            const float xx = (h & 1) ? bf16hi(w4[h / 2]) : bf16lo(w4[h / 2]);
            const bool k = fabsf(xx) >= a.tau_x;
            bits |= (k ? 1u : 0u) << h;
            if (k) {
                mx[0][t] = fmaxf(mx[0][t], fabsf(xx * sus[h]));
                mx[1][t] = fmaxf(mx[1][t], fabsf(xx * sgs[h]));
            }
        }
        if (!own || t >= a.nb) bits = 0;
        kb[t] = bits;
        ub |= bits;
        if (a.mask_x && blockIdx.x == 0 && own && t < a.nb) {
            uint32_t lo = 0, hi = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                lo |= ((bits >> b) & 1u) << (8 * b);
                hi |= ((bits >> (b + 4)) & 1u) << (8 * b);
            }
            *reinterpret_cast<uint2 *>(a.mask_x + (size_t)t * a.d + tid * 8) = make_uint2(lo, hi);
        }
    }
    const int cnt = __popc(ub);
    // (2) one block-wide pass: ranks of the kept rows and the maxima
    int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int t = 0; t < B; ++t) {
            float v = mx[m][t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == 0) s_wmax[wid][m * B + t] = v;
        }
    if (lane == 31) s_warp[wid] = inc;
    __syncthreads();
    int base = 0, kx = 0;
#pragma unroll
    for (int w = 0; w < kT / 32; ++w) {
        if (w < wid) base += s_warp[w];
        kx += s_warp[w];
    }
    const int woffs = base + inc - cnt;       // rank of this thread's first kept row
    if (tid < 2 * B) {
        float v = 0.f;
        for (int w = 0; w < kT / 32; ++w) v = fmaxf(v, s_wmax[w][tid]);
        // max |v| < 2^27: v = round(x scale 2^F) fits the four digits
        (&s_F[0][0])[(tid / B) * 4 + tid % B] = v > 0.f ? 26 - ilogbf(v) : 0;
    }
    __syncthreads();
    const int lo = (int)((long long)kx * r / nr);
    const int hi = (int)((long long)kx * (r + 1) / nr);
    const int n_units = hi - lo;
    const int nks = (n_units + kKS - 1) / kKS;

    // (3) the CTA's rows: row index and the digits of x_i scale_i 2^F per
    // (proxy, token); the digit sums of the CTA's rows go to s_S (one
    // (proxy, token) at a time, to keep few registers live)
    const uint32_t dig_m = (L.rowidx - L.dig) / 2;   // bytes of one proxy's digits
    const bool mine = woffs < hi && woffs + cnt > lo;
    if (mine) {
        int rank = woffs;
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            if (!((ub >> h) & 1u)) continue;
            if (rank >= lo && rank < hi) rowidx[rank - lo] = tid * 8 + h;
            ++rank;
        }
    }
#pragma unroll
    for (int t = 0; t < B; ++t)
#pragma unroll 1
    for (int m = 0; m < 2; ++m) {
        int ds0 = 0, ds1 = 0, ds2 = 0, ds3 = 0;
        if (mine) {
            const int F = s_F[m][t];
            const float sc1 = __int_as_float((127 + F / 2) << 23);
            const float sc2 = __int_as_float((127 + F - F / 2) << 23);
            unsigned char *dm = sm + L.dig + (uint32_t)m * dig_m;
            const uint32_t xw[4] = {xv[t].x, xv[t].y, xv[t].z, xv[t].w};
            int rank = woffs;
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                if (!((ub >> h) & 1u)) continue;
                if (rank >= lo && rank < hi) {
                    const int u = rank - lo;
                    const float xx = ((kb[t] >> h) & 1u) ? ((h & 1) ? bf16hi(xw[h / 2]) : bf16lo(xw[h / 2]))
                                                         : 0.f;
                    const int v = __float2int_rn(xx * (m ? sgs[h] : sus[h]) * sc1 * sc2);
                    const int d3 = v >> 21;
                    const int rr = v - d3 * (1 << 21);
                    const int d0 = rr & 127, d1 = (rr >> 7) & 127, d2 = rr >> 14;
                    dm[dig_off(u, 4 * t + 0)] = (unsigned char)d0;
                    dm[dig_off(u, 4 * t + 1)] = (unsigned char)d1;
                    dm[dig_off(u, 4 * t + 2)] = (unsigned char)d2;
                    dm[dig_off(u, 4 * t + 3)] = (unsigned char)d3;
                    ds0 += d0;
                    ds1 += d1;
                    ds2 += d2;
                    ds3 += d3;
                }
                ++rank;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ds0 += __shfl_xor_sync(0xffffffffu, ds0, o);
            ds1 += __shfl_xor_sync(0xffffffffu, ds1, o);
            ds2 += __shfl_xor_sync(0xffffffffu, ds2, o);
            ds3 += __shfl_xor_sync(0xffffffffu, ds3, o);
        }
        if (lane == 0 && (ds0 | ds1 | ds2 | ds3)) {
            atomicAdd(&s_S[m][t][0], ds0);
            atomicAdd(&s_S[m][t][1], ds1);
            atomicAdd(&s_S[m][t][2], ds2);
            atomicAdd(&s_S[m][t][3], ds3);
        }
    }
    fence_async_smem();  // the digits are read by the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) stamp_max(a.stamps, kS1Pro);
    const uint32_t tmem = s_tmem;

    if (wid < kDecW) {
        // ---------------- loads and decode into the A tiles ----------------
        // piece tid of every K step: row k, proxy m, 16-byte piece p of the
        // row's 128-byte granule (channels 32p .. 32p + 31 of the block)
        const int k = tid >> 4, m = (tid >> 3) & 1, p = tid & 7;
        const uint8_t *qb = (m ? a.q_gate : a.q_up) + (size_t)c0 * a.d * 128 + p * 16;
        const uint64_t pol = l2_evict_first();
        const uint32_t toff = (uint32_t)(m * 2 + (p >> 2)) * kATile + (uint32_t)(k >> 3) * 1024u +
                              (uint32_t)(k & 7) * 128u;
        const uint32_t off_lo = toff + ((uint32_t)((2 * (p & 3)) ^ (k & 7)) << 4);
        const uint32_t off_hi = toff + ((uint32_t)((2 * (p & 3) + 1) ^ (k & 7)) << 4);
        uint4 buf[kPre];
#pragma unroll
        for (int i = 0; i < kPre; ++i) {
            const int u = i * kKS + k;
            buf[i] = make_uint4(0u, 0u, 0u, 0u);
            if (u < n_units) buf[i] = ldg16(qb + (size_t)rowidx[u] * 128, pol);
        }
        bool ok = true;
        for (int ks0 = 0; ks0 < nks && ok; ks0 += kPre) {
#pragma unroll
            for (int i = 0; i < kPre; ++i) {
                const int ks = ks0 + i;
                if (ks >= nks) break;
                const uint4 w = buf[i];
                const int un = (ks + kPre) * kKS + k;
                buf[i] = make_uint4(0u, 0u, 0u, 0u);
                if (un < n_units) buf[i] = ldg16(qb + (size_t)rowidx[un] * 128, pol);
                const int as = ks % kASlots;
                // the slot is free once the MMAs of K step ks - kASlots are done
                if (ks >= kASlots &&
                    !__all_sync(0xffffffffu, s1_wait(&a_empty[as], ((ks / kASlots) - 1) & 1, a, &s_fail))) {
                    ok = false;
                    break;
                }
                unsigned char *ab = sm + L.a + as * kAStep;
                *reinterpret_cast<uint4 *>(ab + off_lo) =
                    make_uint4(w.x & 0x0F0F0F0Fu, w.y & 0x0F0F0F0Fu, w.z & 0x0F0F0F0Fu, w.w & 0x0F0F0F0Fu);
                *reinterpret_cast<uint4 *>(ab + off_hi) =
                    make_uint4(w.x & 0xF0F0F0F0u, w.y & 0xF0F0F0F0u, w.z & 0xF0F0F0F0u, w.w & 0xF0F0F0F0u);
                fence_async_smem();
                __syncwarp();
                // test hook: in CTA 0 warp 0 never completes this K step
                if (lane == 0 && !(a.debug_skip == ks && blockIdx.x == 0 && wid == 0))
                    mbar_arrive(&a_full[as]);
            }
        }
    } else if (wid == kMmaW) {
        // ---------------- MMA issue ----------------
        if (lane == 0) {
            for (int ks = 0; ks < nks; ++ks) {
                const int as = ks % kASlots;
                if (!s1_wait(&a_full[as], (ks / kASlots) & 1, a, &s_fail)) break;
                tc_fence_after();
                const uint32_t kb_off = (uint32_t)(ks >> 2) * 2048u + (uint32_t)(ks & 3) * 32u;
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const uint64_t db = sw128_desc(sbase + L.dig + m * dig_m + kb_off, 16, 1024);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
                        umma_i8(tmem + (m * 2 + mt) * kN,
                                sw128_desc(sbase + L.a + as * kAStep + (m * 2 + mt) * kATile, 4096, 1024),
                                db, kIdesc, ks > 0 ? 1u : 0u);
                }
                umma_commit(&a_empty[as]);
            }
            umma_commit(done);  // every MMA issued above is complete
        }
        __syncwarp();
    }

    // ---------------- epilogue: the CTA's exact partials ----------------
    long long *acc = reinterpret_cast<long long *>(a.acc);
    if (wid < kDecW) {
        // done's single phase completes once the MMA thread's last commit
        // lands (it commits even after giving up, so no MMA is left running
        // when tensor memory is read and freed; bounded by the default limit,
        // not by the shortened test limit)
        const bool ok = mbar_wait(done, 0, kDefaultWaitUs);
        if (!ok && lane == 0) atomicOr(a.status, kStTimeoutRing);
        tc_fence_after();
        const int q = wid & 3, pair = wid >> 2;  // lane quadrant, (proxy, M tile)
        const int m = pair >> 1, mt = pair & 1;
        uint32_t D[kN];
#pragma unroll
        for (int n = 0; n < kN; ++n) D[n] = 0u;
        if (nks > 0 && ok) tmem_ld16(tmem + (uint32_t)pair * kN + ((uint32_t)(q * 32) << 16), D);
        const int mi = q * 32 + lane;          // M row of the tile
        const int rr = mi & 31;
        const bool odd = rr >= 16;
        const int ch = mt * 128 + (mi & ~31) + (odd ? 2 * (rr - 16) + 1 : 2 * rr);
#pragma unroll
        for (int t = 0; t < B; ++t) {
            if (t >= a.nb) break;
            long long V = 0;
#pragma unroll
            for (int l = 0; l < 4; ++l) {
                const int dl = odd ? ((int)D[4 * t + l] >> 4) : (int)D[4 * t + l];
                V += ((long long)dl - 8ll * s_S[m][t][l]) * (1ll << (7 * l));
            }
            if (V) atomicAdd(reinterpret_cast<unsigned long long *>(
                                 acc + ((size_t)(m * B + t) * a.f + (size_t)c0 * kCB + ch)),
                             (unsigned long long)V);
        }
        __threadfence();  // the partials are in L2 before this CTA is counted
    }
    if (tid == 0) stamp_max(a.stamps, kS1Stream);
    tc_fence_before();
    __syncthreads();
    if (wid == kMmaW) {
        tc_fence_after();
        tmem_free(tmem, 64);
    }
    if (tid == 0) {
        const int prev = atomicAdd(a.blk_cnt + c0, 1);
        s_last = (prev == nr - 1);
        __threadfence();
    }
    __syncthreads();
    if (s_last) {
        if (tid == 0) stamp_max(a.stamps, kS1Red);
        // (4) the last CTA of the block: exact sums -> s~ -> masks and lists
        const int ch = tid;                    // channel within the block
        const int j = c0 * kCB + ch;
        uint32_t bits = 0;
        if (ch < kCB) {
#pragma unroll
            for (int t = 0; t < B; ++t) {
                if (t >= a.nb) break;
                long long *pu = acc + ((size_t)(0 * B + t) * a.f + j);
                long long *pg = acc + ((size_t)(1 * B + t) * a.f + j);
                const long long Vu = __ldcg(pu), Vg = __ldcg(pg);
                const float uu = (float)ldexp((double)Vu, -s_F[0][t]);
                const float gg = (float)ldexp((double)Vg, -s_F[1][t]);
                const float st = uu * gate_act(gg, a.act);
                if (a.s_out) a.s_out[(size_t)t * a.f + j] = st;
                const bool keep = fabsf(st) >= a.tau_s;
                if (a.mask_s) a.mask_s[(size_t)t * a.f + j] = keep ? 1 : 0;
                bits |= (keep ? 1u : 0u) << t;
            }
        }
        if (a.build_lists) {
            // warp ballots and per-warp counts (token t in column t, union in
            // column B). A one-token pass writes only the union list and
            // count: they are the token's (Stage 2 reads them for both).
            constexpr int T0 = B == 1 ? 1 : 0;
            uint32_t bal[B + 1];
#pragma unroll
            for (int t = T0; t <= B; ++t) {
                const bool k = (t < B) ? ((bits >> t) & 1u) : (bits != 0u);
                bal[t] = __ballot_sync(0xffffffffu, k);
                if (lane == 0) s_cnt[wid][t] = __popc(bal[t]);
            }
            __syncthreads();
            const uint32_t lt = (1u << lane) - 1u;
            constexpr int WPB = kCB / 32;
            if (wid < WPB) {
#pragma unroll
                for (int t = T0; t <= B; ++t) {
                    int bse = 0, tot = 0;
                    for (int w = 0; w < WPB; ++w) {
                        if (w < wid) bse += s_cnt[w][t];
                        tot += s_cnt[w][t];
                    }
                    const bool k = (bal[t] >> lane) & 1u;
                    const int pos = bse + __popc(bal[t] & lt);
                    if (t < B) {
                        if (k) a.tlist[(size_t)t * a.f + c0 * kCB + pos] = j;
                        if (tid == 0) a.tcount[c0 * B + t] = (t < a.nb) ? tot : 0;
                    } else {
                        if (k) a.ulist[(size_t)c0 * kCB + pos] = (uint32_t)j | (bits << 24);
                        if (tid == 0) a.ucount[c0] = tot;
                    }
                }
            }
        }
    }
    if (a.stamps) {  // uniform over the grid
        __syncthreads();
        if (tid == 0) stamp_max(a.stamps, kS1End);
    }
}

template <int B>
cudaError_t launch_tc(const Stage1Args &a, int grid, size_t smem, cudaStream_t s) {
    auto k = k_stage1_tc<B>;
    cudaError_t e = set_max_dynamic_smem((const void *)k, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3(grid), dim3(kT), smem, s, a);
}

}  // namespace

// Plan of the tensor-core Stage 1 for passes of <= 4 tokens; false if the
// shape is outside what it handles (d_model <= 4096: one 8-coordinate chunk
// per thread; shared memory within the budget)
bool stage1_tc_plan(int d, int f, int B, int sms, int *n_r, int *unit_cap, size_t *smem) {
    if (B > 4 || d > 8 * kT || d % 8) return false;
    const int C = f / kCB;
    int nr = sms / C;
    if (nr > 8) nr = 8;
    if (nr < 1) nr = 1;
    const int cap = (d + nr - 1) / nr;
    const size_t sz = tc_smem(cap).total;
    if (sz > (size_t)kS2SmemBudget) return false;
    *n_r = nr;
    *unit_cap = cap;
    *smem = sz;
    return true;
}

cudaError_t launch_stage1_tc(int B, const Stage1Args &a, size_t smem, cudaStream_t s) {
    const int grid = a.C * a.n_r;
    if (B == 1) return launch_tc<1>(a, grid, smem, s);
    if (B == 2) return launch_tc<2>(a, grid, smem, s);
    if (B == 4) return launch_tc<4>(a, grid, smem, s);
    return cudaErrorInvalidValue;
}

}  // namespace prox
