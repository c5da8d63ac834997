// Stage 1 of the Prox sparse SwiGLU FFN on sm_100a: input mask, input-sparse
// INT4 proxy GEMVs for up and gate, proxy state and the shared channel mask
// (Prox deep-dive blog, section "Stage 1"; input-sparse projection Pi_in of
// the translated arXiv page, section 2.2).
//
// Layout. The proxies are block-tiled: q[c][i][0..127] holds the 256 channels
// [256c, 256c + 256) of input row i, two per byte. A rejected input
// coordinate skips one 128-byte granule per block, and the kept rows of one
// block are adjacent granules of one d_model * 128-byte region.
//
// Work split. Column block c (256 channels) is handled by a thread-block
// cluster of n_r CTAs; CTA r of the cluster takes the r-th contiguous range
// of the kept rows (ranks over the union of the pass's tokens) and streams
// the granules of BOTH proxies (one read of x serves up and gate, the fused
// split-N kernel of the blog's "From formula to GPU" section). Each thread
// keeps two sets of rows of its 16/8/4-byte chunk in flight in registers
// (load one set while decoding the other), about 64 KB per CTA. The cluster's
// partial sums meet in distributed shared memory: CTA 0 adds them in rank
// order, forms s~ = u~ * SiLU(g~), thresholds it and compacts the kept
// channels into ascending lists, so the result is deterministic.
//
// INT4 decode. A nibble n at bits 4p..4p+3 of a word, with every other bit
// cleared, is the bit pattern of the subnormal float n * 2^(4p-149). One XOR
// of the whole word with 0x88888888 turns every stored two's complement code q
// into n = q + 8, then one AND per weight yields an exact float operand; the FMA multiplies it by x_i * scale_i pre-scaled by
// 2^E (E chosen per CTA so sums stay normal). At the end each channel's sum
// is rescaled by the exact power of two 2^(149 - 4p - E) and the offset
// 8 * sum(x_i * scale_i) is removed. Nibbles 5..7 of a word are first shifted
// down by 12 bits (to positions 2..4). Subnormal operands need FMA without
// flush-to-zero, which is the default without fast-math.
#include "prox_internal.cuh"

#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace cg = cooperative_groups;

namespace prox {
namespace {

template <int B, int NB>
struct S1 {
    static constexpr int CW = NB * kCB;                              // channels per CTA
    // channels per thread; every warp covers whole rows of one row lane
    static constexpr int CPT = (B == 1 && NB == 2) ? 32 : (B <= 4 ? 16 : 8);
    static constexpr int BYTES = CPT / 2;                            // bytes per row per thread
    static constexpr int WORDS = BYTES / 4;
    static constexpr int ACC = B * CPT;
    static constexpr int TPRB = kCB / CPT;                           // threads per block per matrix
    static constexpr int TPRM = CW / CPT;                            // threads per row per matrix
    static constexpr int TPR = 2 * TPRM;                             // threads per row
    static constexpr int RL = kS1Threads / TPR;                      // row lanes
    static constexpr int U = (B >= 4 ? 8 : 16) / WORDS;              // rows per load set
};

template <int WORDS>
struct Vec {
    uint32_t w[WORDS];
};

// streaming 16/8/4-byte load that does not allocate in L1
__device__ __forceinline__ void ld_stream(Vec<4> &v, const uint8_t *p) {
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3])
                 : "l"(p));
}
__device__ __forceinline__ void ld_stream(Vec<2> &v, const uint8_t *p) {
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(v.w[0]), "=r"(v.w[1])
                 : "l"(p));
}
__device__ __forceinline__ void ld_stream(Vec<1> &v, const uint8_t *p) {
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v.w[0]) : "l"(p));
}

// nibble position (in units of 4 bits) of local channel k of a word after
// the decode above
__host__ __device__ constexpr int nib_pos(int k) { return k < 5 ? k : k - 3; }

// nibble p of a word already XOR-ed with 0x88888888, as a subnormal float
__device__ __forceinline__ float nib_f(uint32_t wx, int p) {
    return __uint_as_float(wx & (0xFu << (4 * p)));
}

// acc2 holds channel pairs: channel t * CPT + wi * 8 + k is component k % 2 of
// acc2[(t * CPT + wi * 8 + k) / 2]; it gains xs[t] * code_k * 2^(4 pos(k) - 149)
template <int B, int CPT>
__device__ __forceinline__ void proc_word(uint32_t w0, int wi, const float *xs, float2 *acc2) {
    const uint32_t w = w0 ^ 0x88888888u;  // every two's complement code q -> q + 8
    const uint32_t v = w >> 12;
    const float2 d01 = make_float2(nib_f(w, 0), nib_f(w, 1));
    const float2 d23 = make_float2(nib_f(w, 2), nib_f(w, 3));
    const float2 d45 = make_float2(nib_f(w, 4), nib_f(v, 2));
    const float2 d67 = make_float2(nib_f(v, 3), nib_f(v, 4));
#pragma unroll
    for (int t = 0; t < B; ++t) {
        const float2 xx = make_float2(xs[t], xs[t]);
        float2 *a = acc2 + (t * CPT + wi * 8) / 2;
        a[0] = __ffma2_rn(xx, d01, a[0]);
        a[1] = __ffma2_rn(xx, d23, a[1]);
        a[2] = __ffma2_rn(xx, d45, a[2]);
        a[3] = __ffma2_rn(xx, d67, a[3]);
    }
}

// deterministic block-wide exclusive scan of one int per thread (256 threads)
__device__ __forceinline__ int block_excl_scan(int v, int *warp_tot, int &total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) warp_tot[wid] = inc;
    __syncthreads();
    int base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kS1Threads / 32; ++w) {
        if (w < wid) base += warp_tot[w];
        tot += warp_tot[w];
    }
    __syncthreads();
    total = tot;
    return base + inc - v;
}

}  // namespace

// shared-memory carve-up of one Stage-1 CTA (kept next to the kernel)
struct S1Smem {
    size_t red, tmask, rowidx, xs, part, total;
};

__host__ __device__ inline S1Smem s1_smem(int d, int B, int NB, int unit_cap) {
    const int cw = NB * kCB;
    const int cpt = (B == 1 && NB == 2) ? 32 : (B <= 4 ? 16 : 8);
    const int rl = kS1Threads / (2 * (cw / cpt));
    const size_t red = (size_t)rl * 2 * B * (cw + cw / cpt) * 4;    // padded row-lane sums
    const int W = d / 32;
    S1Smem s;
    size_t o = 0;
    s.red = o;
    o += red;
    s.tmask = o;
    o += (size_t)B * W * 4;
    s.rowidx = o;
    o += (size_t)unit_cap * 4;
    s.xs = o;
    o += (size_t)unit_cap * 2 * B * 4;
    s.part = o;
    o += (size_t)2 * B * cw * 4;
    s.total = o;
    return s;
}

namespace {

template <int B, int NB>
__global__ void __launch_bounds__(kS1Threads, 1) k_stage1(const Stage1Args a) {
    using T = S1<B, NB>;
    extern __shared__ __align__(16) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    cg::cluster_group cluster = cg::this_cluster();
    const int r = (int)cluster.block_rank();  // row group
    const int c0 = (blockIdx.x / a.n_r) * NB;  // first column block of the group
    const int W = a.d / 32;                    // mask words per token
    const S1Smem L = s1_smem(a.d, B, NB, a.unit_cap);
    float *red = reinterpret_cast<float *>(smem + L.red);
    uint32_t *tmask = reinterpret_cast<uint32_t *>(smem + L.tmask);  // [B][W]
    int *rowidx = reinterpret_cast<int *>(smem + L.rowidx);          // [unit_cap]
    float *xs = reinterpret_cast<float *>(smem + L.xs);              // [unit_cap][2][B]
    float *part = reinterpret_cast<float *>(smem + L.part);          // [2][B][CW]
    __shared__ int s_warp[kS1Threads / 32];
    __shared__ float s_red[kS1Threads / 32][4 * kMaxB];
    __shared__ int s_E[kMaxB];
    __shared__ int s_cnt[kS1Threads / 32][kMaxB + 1];

    // Programmatic dependent launch: x, y and the workspace may belong to the
    // previous kernel in the stream; wait for it, then let the next kernel
    // (Stage 2) start its own prologue.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    // (1) Stage 2 accumulates y with atomics: clear it here.
    if (a.y_zero) {
        float4 *y4 = reinterpret_cast<float4 *>(a.y_zero);
        const int n4 = a.nb * a.d / 4;
        for (int k = blockIdx.x * kS1Threads + tid; k < n4; k += gridDim.x * kS1Threads)
            y4[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // (2) input masks m_x = 1[|x_i| >= tau_x] per token: each thread owns
    // 16-byte chunks of 8 coordinates; all its loads are issued before any
    // use. Chunk ci's 8 keep bits are byte ci of the token's mask words. The
    // same pass finds max |x| per token, which fixes the power-of-two
    // pre-scale 2^E (see the decode note above).
    {
        // chunks per thread per token (d_model <= 8192; <= 4096 when B = 8)
        constexpr int MAXK = (B == 8 ? 4096 : 8192) / 8 / kS1Threads;
        const int NC = a.d / 8;
        uint4 xv[MAXK][B];
#pragma unroll
        for (int k = 0; k < MAXK; ++k)
#pragma unroll
            for (int t = 0; t < B; ++t) {
                const int ci = tid + k * kS1Threads;
                xv[k][t] = make_uint4(0, 0, 0, 0);
                if (ci < NC && t < a.nb)
                    xv[k][t] = *reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.d + ci * 8);
            }
        uint8_t *tbytes = reinterpret_cast<uint8_t *>(tmask);
        float xmax[B];
#pragma unroll
        for (int t = 0; t < B; ++t) xmax[t] = 0.f;
#pragma unroll
        for (int k = 0; k < MAXK; ++k) {
            const int ci = tid + k * kS1Threads;
            if (ci >= NC) break;
#pragma unroll
            for (int t = 0; t < B; ++t) {
                const uint32_t w4[4] = {xv[k][t].x, xv[k][t].y, xv[k][t].z, xv[k][t].w};
                uint32_t bits = 0;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float lo = fabsf(bf16lo(w4[h])), hi = fabsf(bf16hi(w4[h]));
                    bits |= (lo >= a.tau_x ? 1u : 0u) << (2 * h);
                    bits |= (hi >= a.tau_x ? 1u : 0u) << (2 * h + 1);
                    xmax[t] = fmaxf(xmax[t], fmaxf(lo, hi));
                }
                if (t >= a.nb) bits = 0;
                tbytes[t * NC + ci] = (uint8_t)bits;
                if (a.mask_x && blockIdx.x == 0 && t < a.nb) {
                    uint32_t lo = 0, hi = 0;
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        lo |= ((bits >> b) & 1u) << (8 * b);
                        hi |= ((bits >> (b + 4)) & 1u) << (8 * b);
                    }
                    *reinterpret_cast<uint2 *>(a.mask_x + (size_t)t * a.d + ci * 8) =
                        make_uint2(lo, hi);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < B; ++t) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                xmax[t] = fmaxf(xmax[t], __shfl_xor_sync(0xffffffffu, xmax[t], o));
            if (lane == 0) s_red[wid][t] = xmax[t];
        }
    }
    __syncthreads();

    // (3) one thread per mask word: union mask, its population, ranks of the
    // kept rows (one block-wide scan) and this CTA's share of them
    if (tid < B) {
        float mx = 0.f;
        for (int w = 0; w < kS1Threads / 32; ++w) mx = fmaxf(mx, s_red[w][tid]);
        // |x * 2^E| < 2^96: a row sum of (q + 8) * x_i * scale_i * 2^E over
        // <= 8192 rows stays finite for scales below 2^15 and, for scales
        // above 2^-70, partial sums of the subnormal-coded products stay normal
        s_E[tid] = (mx > 0.f) ? 95 - ilogbf(mx) : 0;
    }
    uint32_t um = 0;
    if (tid < W) {
#pragma unroll
        for (int t = 0; t < B; ++t) um |= tmask[t * W + tid];
    }
    int kx;
    const int woffs = block_excl_scan(__popc(um), s_warp, kx);  // syncs the CTA
    const int lo = (int)((long long)kx * r / a.n_r);
    const int hi = (int)((long long)kx * (r + 1) / a.n_r);
    const int n_units = hi - lo;
    if (woffs < hi && woffs + __popc(um) > lo) {
        int rank = woffs;
        for (uint32_t b = um; b; b &= b - 1, ++rank)
            if (rank >= lo && rank < hi) rowidx[rank - lo] = tid * 32 + (__ffs(b) - 1);
    }
    __syncthreads();

    // Each thread streams rows u = rl, rl + RL, ... (its k-th row is u =
    // rl + k * RL) of one 16/8/4-byte chunk of one proxy's granules.
    const int rl = tid / T::TPR;
    const int m = (tid / T::TPRM) & 1;
    const int chunk = tid % T::TPRM;
    const uint8_t *gsrc = (m ? a.q_gate : a.q_up) +
                          (size_t)(c0 + chunk / T::TPRB) * a.d * (kCB / 2) +
                          (chunk % T::TPRB) * T::BYTES;
    const int n_rows = n_units > rl ? (n_units - rl + T::RL - 1) / T::RL : 0;
    Vec<T::WORDS> va[T::U], vb[T::U];
    auto load_set = [&](Vec<T::WORDS>(&v)[T::U], int k0) {
#pragma unroll
        for (int j = 0; j < T::U; ++j)
            if (k0 + j < n_rows)
                ld_stream(v[j], gsrc + (size_t)rowidx[rl + (k0 + j) * T::RL] * (kCB / 2));
    };

    // (4) x_i * scale_i * 2^E per matrix and token for the units (exact
    // power-of-two scaling, split in two factors so each is a normal float).
    // The few gather loads go out first, the first two row sets right after.
    {
        float pe1[B], pe2[B];
#pragma unroll
        for (int t = 0; t < B; ++t) {
            const int e1 = s_E[t] / 2, e2 = s_E[t] - e1;
            pe1[t] = __int_as_float((127 + e1) << 23);
            pe2[t] = __int_as_float((127 + e2) << 23);
        }
        constexpr int G4 = 2;  // units per thread per batch of loads
        bool started = false;
        for (int u0 = tid; u0 < n_units || !started; u0 += G4 * kS1Threads) {
            float su[G4], sg[G4];
            uint16_t xh[G4][B];
#pragma unroll
            for (int k = 0; k < G4; ++k) {
                const int u = u0 + k * kS1Threads;
                su[k] = sg[k] = 0.f;
                if (u < n_units) {
                    const int i = rowidx[u];
                    su[k] = a.s_up[i];
                    sg[k] = a.s_gate[i];
#pragma unroll
                    for (int t = 0; t < B; ++t)
                        xh[k][t] = (t < a.nb) ? a.x[(size_t)t * a.d + i] : (uint16_t)0;
                }
            }
            if (!started) {
                load_set(va, 0);
                load_set(vb, T::U);
                started = true;
            }
#pragma unroll
            for (int k = 0; k < G4; ++k) {
                const int u = u0 + k * kS1Threads;
                if (u >= n_units) break;
                const int i = rowidx[u];
#pragma unroll
                for (int t = 0; t < B; ++t) {
                    float xv = 0.f;
                    if ((tmask[t * W + (i >> 5)] >> (i & 31)) & 1u)
                        xv = __uint_as_float((uint32_t)xh[k][t] << 16);
                    xs[(u * 2 + 0) * B + t] = (xv * su[k]) * pe1[t] * pe2[t];
                    xs[(u * 2 + 1) * B + t] = (xv * sg[k]) * pe1[t] * pe2[t];
                }
            }
        }
    }
    __syncthreads();

    // (5) main loop: decode one register set while the other is in flight;
    // ssum collects this thread's sum of x_i * scale_i * 2^E (+8 code offset)
    float2 acc2[T::ACC / 2];
#pragma unroll
    for (int k = 0; k < T::ACC / 2; ++k) acc2[k] = make_float2(0.f, 0.f);
    float ssum[B];
#pragma unroll
    for (int t = 0; t < B; ++t) ssum[t] = 0.f;
    auto comp_set = [&](const Vec<T::WORDS>(&v)[T::U], int k0) {
#pragma unroll
        for (int j = 0; j < T::U; ++j) {
            if (k0 + j >= n_rows) break;
            const int u = rl + (k0 + j) * T::RL;
            float xv[B];
#pragma unroll
            for (int t = 0; t < B; ++t) {
                xv[t] = xs[(u * 2 + m) * B + t];
                ssum[t] += xv[t];
            }
#pragma unroll
            for (int q = 0; q < T::WORDS; ++q) proc_word<B, T::CPT>(v[j].w[q], q, xv, acc2);
        }
    };
    for (int k0 = 0; k0 < n_rows; k0 += 2 * T::U) {
        comp_set(va, k0);
        load_set(va, k0 + 2 * T::U);
        comp_set(vb, k0 + T::U);
        load_set(vb, k0 + 3 * T::U);
    }
    __syncthreads();

    // (6) reduce row lanes (padded rows: conflict-free both ways), undo the
    // pre-scale and the +8 code offset: this CTA's partial sums in `part`.
    // The pad word after chunk 0's channels carries the row lane's offset sum.
    constexpr int PAD = T::CW + T::TPRM;  // one extra word per chunk row
#pragma unroll
    for (int t = 0; t < B; ++t) {
        float *row = red + ((rl * 2 + m) * B + t) * PAD;
#pragma unroll
        for (int k = 0; k < T::CPT; k += 2) {
            row[chunk * (T::CPT + 1) + k] = acc2[(t * T::CPT + k) / 2].x;
            row[chunk * (T::CPT + 1) + k + 1] = acc2[(t * T::CPT + k) / 2].y;
        }
        if (chunk == 0) row[T::CPT] = ssum[t];
    }
    __syncthreads();
    for (int o = tid; o < 2 * T::CW; o += kS1Threads) {
        // (matrix, channel within the CTA's columns)
        const int mm = o / T::CW, ch = o % T::CW;
        const int p = nib_pos(ch % 8);
        const int pos = (ch / T::CPT) * (T::CPT + 1) + ch % T::CPT;
        // 2^(149 - 4p) and 2^-E as products of normal floats
        const float up1 = __int_as_float((127 + 75) << 23);
        const float up2 = __int_as_float((127 + 74 - 4 * p) << 23);
#pragma unroll
        for (int t = 0; t < B; ++t) {
            float sacc = 0.f, soff = 0.f;
            for (int q = 0; q < T::RL; ++q) {
                const float *row = red + ((q * 2 + mm) * B + t) * PAD;
                sacc += row[pos];
                soff += row[T::CPT];
            }
            const int e1 = s_E[t] / 2, e2 = s_E[t] - e1;
            const float v = (sacc * up1) * up2 - 8.f * soff;  // sum (q + 8 - 8) x s 2^E
            part[(mm * B + t) * T::CW + ch] =
                v * __int_as_float((127 - e1) << 23) * __int_as_float((127 - e2) << 23);
        }
    }
    cluster.sync();  // all partials of the block are in their CTAs' shared memory

    if (r == 0) {
        // (7) CTA 0 of the cluster: gather the cluster's partials (in rank
        // order), release the peers, then s~ = u~ * SiLU(g~),
        // m_s = 1[|s~| >= tau_s] and the ascending compaction per token and of
        // the union (thread = channel)
        const int ch = tid;                  // channel within the CTA's columns
        const int j = c0 * kCB + ch;         // channel index
        const int blk = wid / (kCB / 32);    // block of this warp's channels
        float uu[B], gg[B];
#pragma unroll(B > 2 ? 1 : B)
        for (int t = 0; t < B; ++t) {
            uu[t] = gg[t] = 0.f;
            if (t >= a.nb || ch >= T::CW) continue;
            // all remote loads first, then the sums in rank order
            float pu[kS1MaxRowGroups], pg[kS1MaxRowGroups];
#pragma unroll
            for (int q = 0; q < kS1MaxRowGroups; ++q) {
                pu[q] = pg[q] = 0.f;
                if (q < a.n_r) {
                    const float *pq = cluster.map_shared_rank(part, q);
                    pu[q] = pq[(0 * B + t) * T::CW + ch];
                    pg[q] = pq[(1 * B + t) * T::CW + ch];
                }
            }
#pragma unroll
            for (int q = 0; q < kS1MaxRowGroups; ++q) {
                uu[t] += pu[q];
                gg[t] += pg[q];
            }
        }
        asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
        uint32_t bits = 0;
#pragma unroll
        for (int t = 0; t < B; ++t) {
            if (t >= a.nb || ch >= T::CW) break;
            const float st = uu[t] * (gg[t] / (1.f + expf(-gg[t])));
            if (a.s_out) a.s_out[(size_t)t * a.f + j] = st;
            const bool keep = fabsf(st) >= a.tau_s;
            if (a.mask_s) a.mask_s[(size_t)t * a.f + j] = keep ? 1 : 0;
            bits |= (keep ? 1u : 0u) << t;
        }
        if (a.build_lists) {
            // warp ballots and per-warp counts (token t in column t, union in column B)
            uint32_t bal[kMaxB + 1];
#pragma unroll
            for (int t = 0; t <= B; ++t) {
                const bool k = (t < B) ? ((bits >> t) & 1u) : (bits != 0u);
                bal[t] = __ballot_sync(0xffffffffu, k);
                if (lane == 0) s_cnt[wid][t] = __popc(bal[t]);
            }
            __syncthreads();
            const uint32_t lt = (1u << lane) - 1u;
            constexpr int WPB = kCB / 32;  // warps per 256-channel block
            if (blk < NB) {
                const int cb = c0 + blk;
#pragma unroll
                for (int t = 0; t <= B; ++t) {
                    int base = 0, tot = 0;
                    for (int w = blk * WPB; w < (blk + 1) * WPB; ++w) {
                        if (w < wid) base += s_cnt[w][t];
                        tot += s_cnt[w][t];
                    }
                    const bool k = (bal[t] >> lane) & 1u;
                    const int pos = base + __popc(bal[t] & lt);
                    const bool first = (wid == blk * WPB) && lane == 0;
                    if (t < B) {
                        if (k) a.tlist[(size_t)t * a.f + cb * kCB + pos] = j;
                        if (first) a.tcount[cb * B + t] = (t < a.nb) ? tot : 0;
                    } else {
                        if (k) a.ulist[(size_t)cb * kCB + pos] = (uint32_t)j | (bits << 24);
                        if (first) a.ucount[cb] = tot;
                    }
                }
            }
        }
        asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    } else {
        // peers keep their shared memory until CTA 0 has gathered it
        asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
        asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    }
}

template <int B, int NB>
cudaError_t launch1(Stage1Args a, const Stage1Plan &p0, cudaStream_t s) {
    auto k = k_stage1<B, NB>;
    const int groups = a.C / NB;  // clusters
    // Cluster size (row groups per block): every cluster of the grid must be
    // resident at once, or the last clusters run as a second wave. Start from
    // the plan's choice and shrink until the occupancy calculator agrees.
    struct Cache {
        int d = 0, C = 0, n_r = 0, cap = 0;
        size_t smem = 0;
    };
    static Cache cache;
    Stage1Plan p = p0;
    if (cache.d == a.d && cache.C == a.C) {
        p.n_r = cache.n_r;
        p.unit_cap = cache.cap;
        p.smem = cache.smem;
    } else {
        // fewest row groups whose rows fit in one CTA's shared memory
        int n_min = 1;
        while (n_min < kS1MaxRowGroups &&
               s1_smem(a.d, B, NB, (a.d + n_min - 1) / n_min).total > (size_t)kS2SmemBudget)
            ++n_min;
        if (p.n_r < n_min) p.n_r = n_min;
        for (;;) {
            p.unit_cap = (a.d + p.n_r - 1) / p.n_r;
            p.smem = s1_smem(a.d, B, NB, p.unit_cap).total;
            cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)p.smem);
            if (e != cudaSuccess) return e;
            if (p.n_r <= n_min) break;
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3(groups * p.n_r);
            q.blockDim = dim3(kS1Threads);
            q.dynamicSmemBytes = p.smem;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = p.n_r;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            q.attrs = at;
            q.numAttrs = 1;
            int active = 0;
            e = cudaOccupancyMaxActiveClusters(&active, k, &q);
            if (e != cudaSuccess) return e;
            if (active >= groups) break;
            --p.n_r;
        }
        cache.d = a.d;
        cache.C = a.C;
        cache.n_r = p.n_r;
        cache.cap = p.unit_cap;
        cache.smem = p.smem;
    }
    a.n_r = p.n_r;
    a.unit_cap = p.unit_cap;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(groups * a.n_r);
    cfg.blockDim = dim3(kS1Threads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = a.n_r;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k, a);
}

}  // namespace

cudaError_t launch_stage1(int B, const Stage1Args &a, const Stage1Plan &p, cudaStream_t s) {
#define PROX_S1(BB, NN) \
    if (B == BB && p.nb_blocks == NN) return launch1<BB, NN>(a, p, s);
    PROX_S1(1, 1) PROX_S1(1, 2) PROX_S1(2, 1) PROX_S1(2, 2)
    PROX_S1(4, 1) PROX_S1(4, 2) PROX_S1(8, 1) PROX_S1(8, 2)
#undef PROX_S1
    return cudaErrorInvalidValue;
}

size_t stage1_smem_bytes(int d_model, int B, int NB, int unit_cap) {
    return s1_smem(d_model, B, NB, unit_cap).total;
}

}  // namespace prox
