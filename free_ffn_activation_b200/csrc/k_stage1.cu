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
// streams its 16/8/4-byte chunk of successive rows through a private ring of
// cp.async shared-memory slots (12 rows deep when shared memory allows),
// about 96 KB in flight per CTA: enough to cover the latency, and the decode
// starts sooner than behind a deeper ring. The cluster's
// partial sums meet in distributed shared memory: CTA 0 adds them in rank
// order, forms s~ = u~ * SiLU(g~), thresholds it and compacts the kept
// channels into ascending lists, so the result is deterministic.
//
// INT4 decode. A nibble n at bits 4p..4p+3 of a word, with every other bit
// cleared, is the bit pattern of the subnormal float n * 2^(4p-149). The codes
// are stored offset-binary (n = q + 8), so one AND per weight yields an exact
// float operand; the FMA multiplies it by x_i * scale_i pre-scaled by
// 2^E (E chosen per CTA so sums stay normal). At the end each channel's sum
// is rescaled by the exact power of two 2^(149 - 4p - E) and the offset
// 8 * sum(x_i * scale_i) is removed. Nibbles 5..7 of a word are first shifted
// down by 12 bits (to positions 2..4). Subnormal operands need FMA without
// flush-to-zero, which is the default without fast-math.
//
// Passes of 4 or 8 tokens with the INT4 proxy can form the proxy products on
// the tensor cores instead (s1_tc_stream below: tcgen05 kind::i8 over the
// codes as bytes and fixed-point digits of x, exact int32 accumulation); the
// prologue, the cluster reduction and the lists are shared.
#include "prox_internal.cuh"
#include "umma.cuh"

#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

namespace cg = cooperative_groups;

namespace prox {
namespace {

// Proxy kinds (PK): 0 = INT4 codes, two per byte (the method's proxy);
// 1 = bf16 weights (the FP16/bf16-proxy ablation of the blog's "Evidence").
// channels per thread: a warp covers whole rows of one row lane
__host__ __device__ constexpr int s1_cpt(int B, int NB, int PK = 0) {
    return PK ? 8 : ((B <= 2 && NB == 2) ? 32 : (B <= 4 ? 16 : 8));
}
// bytes of one row a thread moves per copy, and bytes of one row of a block
__host__ __device__ constexpr int s1_bytes(int B, int NB, int PK) {
    return PK ? 16 : s1_cpt(B, NB) / 2;
}
__host__ __device__ constexpr int s1_gran(int PK) { return PK ? kCB * 2 : kCB / 2; }
// deepest per-thread ring (rows in flight) and the ring bytes it takes
__host__ __device__ constexpr int s1_ring_bytes(int B) { return B <= 2 ? 192 : (B == 4 ? 256 : 128); }
__host__ __device__ constexpr int s1_dmax(int B, int NB, int PK = 0) {
    return s1_ring_bytes(B) / s1_bytes(B, NB, PK) < 32 ? s1_ring_bytes(B) / s1_bytes(B, NB, PK)
                                                        : 32;
}

template <int B, int NB, int PK = 0>
struct S1 {
    static constexpr int CW = NB * kCB;                              // channels per CTA
    static constexpr int CPT = s1_cpt(B, NB, PK);                    // channels per thread
    static constexpr int BYTES = s1_bytes(B, NB, PK);                // bytes per row per thread
    static constexpr int GRAN = s1_gran(PK);                         // bytes per row per block
    static constexpr int WORDS = BYTES / 4;
    static constexpr int ACC = B * CPT;
    static constexpr int TPRB = kCB / CPT;                           // threads per block per matrix
    static constexpr int TPRM = CW / CPT;                            // threads per row per matrix
    static constexpr int TPR = 2 * TPRM;                             // threads per row
    static constexpr int RL = kS1Threads / TPR;                      // row lanes
    static constexpr int DMAX = s1_dmax(B, NB, PK);                  // deepest ring (rows)
    static constexpr int KMAX = (B == 8 ? 4096 : 8192) / 8 / kS1Threads;  // x chunks per thread
};

// cp.async of BYTES (16, 8 or 4) from global to shared under L2 policy pol;
// 16-byte copies skip L1
template <int BYTES>
__device__ __forceinline__ void cp_async(void *dst, const void *src, uint64_t pol) {
    if constexpr (BYTES == 16) {
        asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(
                         smem_addr(dst)),
                     "l"(src), "l"(pol)
                     : "memory");
    } else {
        asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], %2, %3;" ::"r"(
                         smem_addr(dst)),
                     "l"(src), "n"(BYTES), "l"(pol)
                     : "memory");
    }
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// nibble position (in units of 4 bits) of local channel k of a word after
// the decode above
__host__ __device__ constexpr int nib_pos(int k) { return k < 5 ? k : k - 3; }

// nibble p of a word of offset-binary codes, as a subnormal float
__device__ __forceinline__ float nib_f(uint32_t wx, int p) {
    return __uint_as_float(wx & (0xFu << (4 * p)));
}

// acc2 holds channel pairs: channel t * CPT + wi * 8 + k is component k % 2 of
// acc2[(t * CPT + wi * 8 + k) / 2]; it gains xs[t] * code_k * 2^(4 pos(k) - 149)
template <int B, int CPT>
__device__ __forceinline__ void proc_word(uint32_t w0, int wi, const float *xs, float2 *acc2) {
    const uint32_t w = w0;  // nibbles hold q + 8
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

// bf16 proxy: word wi of a thread's 16-byte chunk holds channels 2 wi (low
// half) and 2 wi + 1 (high half); acc2[(t * CPT + 2 wi) / 2] gains xs[t] * w
template <int B, int CPT>
__device__ __forceinline__ void proc_word_bf16(uint32_t w, int wi, const float *xs, float2 *acc2) {
    const float2 dw = make_float2(bf16lo(w), bf16hi(w));
#pragma unroll
    for (int t = 0; t < B; ++t) {
        const float2 xx = make_float2(xs[t], xs[t]);
        float2 *a = acc2 + (t * CPT + wi * 2) / 2;
        a[0] = __ffma2_rn(xx, dw, a[0]);
    }
}

// deterministic block-wide exclusive scan of one int per thread (one
// barrier; warp_tot is written once per kernel, so it needs no second one)
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
    total = tot;
    return base + inc - v;
}

}  // namespace

// Tensor-core proxy products (passes of 4 or 8 tokens, INT4 proxy): shared
// memory of the stream, which replaces the copy ring and row-lane reduction
// area: two K steps of decoded codes for both matrices and the digits of x.
constexpr int kTcKStep = 32;   // proxy rows per K step (the K of one kind::i8 MMA)
// K steps decoded per group (one group of codes in flight per thread)
__host__ __device__ constexpr int s1tc_group(int NB) { return NB == 2 ? 2 : 3; }
__host__ __device__ inline size_t s1tc_bytes(int B, int NB, int unit_cap) {
    const size_t a = (size_t)s1tc_group(NB) * 2 * kTcKStep * NB * kCB;     // group x 2 matrices
    const size_t b = (size_t)2 * ((unit_cap + 127) / 128) * (4 * B / 8) * 1024;  // digits
    return 1024 + a + b;                                                   // + alignment slack
}

// shared-memory carve-up of one Stage-1 CTA (kept next to the kernel). The
// copy ring (depth DMAX >> depth_sel rows per thread) and the row-lane
// reduction area are used one after the other and share one region.
struct S1Smem {
    size_t ring, red, rowidx, xs, part, total;
};


__host__ __device__ inline S1Smem s1_smem(int d, int B, int NB, int unit_cap, int depth_sel,
                                         int n_r = kS1MaxRowGroups, int PK = 0, int TC = 0) {
    const int cw = NB * kCB;
    const int cpt = s1_cpt(B, NB, PK);
    const int rl = kS1Threads / (2 * (cw / cpt));
    // row-lane sums: 32-channel chunks swizzled in 16-byte units, narrower
    // chunks padded by one word
    const size_t red = (size_t)rl * 2 * B * (cpt == 32 ? cw : cw + cw / cpt) * 4;
    const size_t ring = (size_t)kS1Threads * (s1_dmax(B, NB, PK) >> depth_sel) * s1_bytes(B, NB, PK);
    (void)d;
    S1Smem s;
    size_t o = 0;
    s.ring = s.red = o;
    // the tensor-core stream uses neither the copy ring nor the row-lane
    // area, only its own tiles
    const size_t region = TC ? s1tc_bytes(B, NB, unit_cap) : (ring > red ? ring : red);
    o += region;
    s.rowidx = o;
    o += ((size_t)unit_cap * 4 + 15) / 16 * 16;
    s.xs = o;
    o += (size_t)unit_cap * 2 * B * 4;
    s.part = o;
    o += (size_t)(B <= 2 ? n_r : 1) * 2 * B * cw * 4;  // B <= 2: every rank's partials
    s.total = o;
    return s;
}

namespace {

// (5) main loop: each thread streams rows u = rl, rl + RL, ... (its k-th row
// is u = rl + k * RL) of one 16/8/4-byte chunk of one proxy's granules
// through a private ring of D shared-memory slots, refilling each slot with
// the row D positions later as soon as its words are decoded. ssum collects
// the thread's sum of x_i * scale_i * 2^E (for the +8 code offset).
template <int B, int NB, int PK, int D>
__device__ __forceinline__ void s1_stream(const uint8_t *qbase, unsigned char *ring,
                                          const int *rowidx, const float *xs, int rl, int m,
                                          int n_rows, float2 *acc2, float *ssum) {
    using T = S1<B, NB, PK>;
    // slot-major ring (ring[slot][thread]): a warp's accesses to one slot are
    // consecutive words, free of bank conflicts
    unsigned char *const myring = ring + (size_t)threadIdx.x * T::BYTES;
    constexpr int SLOT = kS1Threads * T::BYTES;  // bytes between a thread's slots
    unsigned char *const ring_end = myring + D * SLOT;
    const uint64_t pol = l2_evict_first();      // each granule is read once per pass
    // walking pointers: the next row to copy, the slot and x of the row to use
    const int *rp = rowidx + rl;
    const float *xp = xs + (rl * 2 + m) * B;
    unsigned char *sp = myring;
    // one copy per loop iteration (no unrolled run of hinted copies)
#pragma unroll 1
    for (int k = 0; k < D; ++k) {
        if (k < n_rows) {
            cp_async<T::BYTES>(myring + k * SLOT, qbase + (size_t)*rp * T::GRAN, pol);
            rp += T::RL;
        }
        cp_commit();
    }
    auto use = [&]() {
        uint32_t w[T::WORDS];
        if constexpr (T::WORDS == 4) {
            const uint4 v = *reinterpret_cast<const uint4 *>(sp);
            w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
        } else if constexpr (T::WORDS == 2) {
            const uint2 v = *reinterpret_cast<const uint2 *>(sp);
            w[0] = v.x; w[1] = v.y;
        } else {
            w[0] = *reinterpret_cast<const uint32_t *>(sp);
        }
        float xv[B];
#pragma unroll
        for (int t = 0; t < B; ++t) {
            xv[t] = xp[t];
            ssum[t] += xv[t];
        }
#pragma unroll
        for (int q = 0; q < T::WORDS; ++q) {
            if constexpr (PK == 0)
                proc_word<B, T::CPT>(w[q], q, xv, acc2);
            else
                proc_word_bf16<B, T::CPT>(w[q], q, xv, acc2);
        }
    };
    // rows 0 .. n_rows - D - 1: each refills its slot with the row D later
    int k = 0;
#pragma unroll 1
    for (; k < n_rows - D; ++k) {
        cp_wait<D - 1>();
        use();
        cp_async<T::BYTES>(sp, qbase + (size_t)*rp * T::GRAN, pol);
        rp += T::RL;
        cp_commit();
        xp += T::RL * 2 * B;
        sp += SLOT;
        if (sp == ring_end) sp = myring;
    }
    // the last D rows (empty groups keep the wait count)
#pragma unroll 1
    for (; k < n_rows; ++k) {
        cp_wait<D - 1>();
        use();
        cp_commit();
        xp += T::RL * 2 * B;
        sp += SLOT;
        if (sp == ring_end) sp = myring;
    }
    cp_wait<0>();
}

// global -> registers, 16 bytes, read-only path, under L2 policy pol
__device__ __forceinline__ uint4 ldg16_pol(const void *src, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(src), "l"(pol));
    return v;
}

// (5'), passes of 4 or 8 tokens with the INT4 proxy: the CTA's proxy rows are
// the K dimension of kind::i8 UMMAs. A = the offset-binary codes q + 8 of one
// matrix as unsigned bytes (MN-major, 128 channels per 128-byte row, 32 rows
// per K step; decoded in registers with two ANDs, a shift and two byte
// permutes per 8 codes). B = x_i * scale_i * 2^E per (matrix, token) as a
// 27-bit fixed-point value v = round(xs * 2^F) split into four signed 8-bit
// digits (v = d0 + 2^7 d1 + 2^14 d2 + 2^21 d3); the digits are the N rows, so
// each code tile is read once for all tokens. D is int32 in TMEM and exact;
// the epilogue removes the +8 offset (8 * the digit sums, exact in int64) and
// undoes 2^F and 2^E: this CTA's partial sums sum_i q_ij x_i scale_i, in the
// same place the CUDA-core stream leaves them. The K steps go in groups of G:
// each thread decodes its codes of the whole group into G tile buffers, makes
// them visible to the tensor core (fence.proxy.async), and only then issues
// the loads of the next group into registers, so no load is outstanding at a
// fence (a fence would wait for it); one CTA barrier and one thread's MMAs
// per group. Waits are bounded.
template <int B, int NB>
__device__ void s1_tc_stream(const Stage1Args &a, unsigned char *region, const int *rowidx,
                             const float *xs, int n_units, const int (&E)[B], int c0,
                             float *part) {
    constexpr int CW = NB * kCB;
    constexpr int N = 4 * B;                          // digit rows
    constexpr int MT = CW / 128;                      // 128-channel M tiles per matrix
    constexpr uint32_t ABUF = 2u * CW * kTcKStep;     // one K step of both matrices
    constexpr uint32_t LBO = (kTcKStep / 8) * 1024u;  // stride of 128-channel atoms
    constexpr uint32_t TCOLS = 2 * MT * N;            // a power of two >= 32
    constexpr uint32_t IDESC = (2u << 4) | (0u << 7) | (1u << 10) | (1u << 15) |
                               ((uint32_t)(N >> 3) << 17) | (8u << 24);  // u8 x s8 -> s32, M 128
    __shared__ float s_mx[2][kMaxB];
    __shared__ int s_F[2][kMaxB];
    __shared__ int s_S[2][kMaxB][4];
    __shared__ uint32_t s_tmem;
    __shared__ __align__(8) uint64_t s_done[2];   // [0]: a group's MMAs, [1]: all MMAs
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const uint32_t rb = (smem_addr(region) + 1023u) & ~1023u;
    constexpr int GR = s1tc_group(NB);                // tile buffers (one group)
    unsigned char *abuf = region + (rb - smem_addr(region));
    unsigned char *bdig = abuf + GR * ABUF;
    const uint32_t aaddr = rb, baddr = rb + GR * ABUF;
    const uint32_t BM = (uint32_t)((a.unit_cap + 127) / 128) * (N / 8) * 1024u;  // one matrix
    const int nks = (n_units + kTcKStep - 1) / kTcKStep;

    if (tid < 2 * kMaxB) (&s_mx[0][0])[tid] = 0.f;
    if (tid < 2 * kMaxB * 4) (&s_S[0][0][0])[tid] = 0;
    if (tid == 0) {
        mbar_init(&s_done[0], 1);
        mbar_init(&s_done[1], 1);
        mbar_fence_init();
    }
    if (wid == 0) tmem_alloc(&s_tmem, TCOLS);
    __syncthreads();
    // fixed-point exponent per (matrix, token): max |xs| * 2^F < 2^27
    {
        float mx[2][B];
#pragma unroll
        for (int mm = 0; mm < 2; ++mm)
#pragma unroll
            for (int t = 0; t < B; ++t) mx[mm][t] = 0.f;
        for (int u = tid; u < n_units; u += kS1Threads)
#pragma unroll
            for (int mm = 0; mm < 2; ++mm)
#pragma unroll
                for (int t = 0; t < B; ++t) mx[mm][t] = fmaxf(mx[mm][t], fabsf(xs[(u * 2 + mm) * B + t]));
#pragma unroll
        for (int mm = 0; mm < 2; ++mm)
#pragma unroll
            for (int t = 0; t < B; ++t) {
                float v = mx[mm][t];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                // non-negative floats order like their bit patterns
                if (lane == 0) atomicMax(reinterpret_cast<int *>(&s_mx[mm][t]), __float_as_int(v));
            }
    }
    __syncthreads();
    if (tid < 2 * B) {
        const float v = s_mx[tid / B][tid % B];
        s_F[tid / B][tid % B] = v > 0.f ? 26 - ilogbf(v) : 0;
    }
    __syncthreads();
    // the digits (B operand, K-major, 128-byte swizzle: 8 digit rows x 128
    // proxy rows per atom); rows past the CTA's units up to the last K step are
    // 0. Thread tid owns the (matrix, token) pair tid % (2B) over every
    // (512 / 2B)-th row and sums its digits in registers; the lanes of a warp
    // that share a pair are reduced with shuffles, so each warp adds 4 counts
    // per pair (integers: the order does not change the sums)
    {
        constexpr int NP = 2 * B;                 // (matrix, token) pairs: 8 or 16
        constexpr int NS = kS1Threads / NP;       // row stripes
        const int pair = tid & (NP - 1), stripe = tid / NP;
        const int mm = pair / B, t = pair % B;
        const int F = s_F[mm][t], f1 = F / 2, f2 = F - f1;
        const float sc1 = __int_as_float((127 + f1) << 23), sc2 = __int_as_float((127 + f2) << 23);
        int dsum[4] = {0, 0, 0, 0};
        for (int u = stripe; u < nks * kTcKStep; u += NS) {
            const int kblk = u >> 7, kin = u & 127;
            int v = 0;
            if (u < n_units) v = __float2int_rn(xs[(u * 2 + mm) * B + t] * sc1 * sc2);
            const int d3 = v >> 21;
            const int r = v - d3 * (1 << 21);
            const int dg[4] = {r & 127, (r >> 7) & 127, r >> 14, d3};
#pragma unroll
            for (int l = 0; l < 4; ++l) {
                const int n = t * 4 + l;
                bdig[mm * BM + (uint32_t)kblk * (N / 8) * 1024u + (n >> 3) * 1024u + (n & 7) * 128u +
                     ((uint32_t)((kin >> 4) ^ (n & 7)) << 4) + (kin & 15)] = (unsigned char)dg[l];
                dsum[l] += dg[l];
            }
        }
#pragma unroll
        for (int l = 0; l < 4; ++l) {
#pragma unroll
            for (int o = NP; o < 32; o <<= 1) dsum[l] += __shfl_xor_sync(0xffffffffu, dsum[l], o);
            if (lane < NP) atomicAdd(&s_S[mm][t][l], dsum[l]);
        }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    // stream: thread tid owns pieces q = tid + 512 j (j < NB) of each K step:
    // 16 bytes (32 channels) of proxy row k of block b of matrix m
    constexpr int G = GR;
    const uint64_t pol = l2_evict_first();
    auto fetch = [&](int ks, uint4 (&dst)[NB]) {
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            const int qq = tid + kS1Threads * j;
            const int piece = qq & 7, k = (qq >> 3) & 31, bm = qq >> 8;
            const int mm = bm & 1, b = bm >> 1;
            const int u = ks * kTcKStep + k;
            dst[j] = make_uint4(0u, 0u, 0u, 0u);
            if (ks < nks && u < n_units)
                dst[j] = ldg16_pol((mm ? a.q_gate : a.q_up) +
                                       ((size_t)(c0 + b) * a.d + rowidx[u]) * (kCB / 2) + piece * 16,
                                   pol);
        }
    };
    uint4 pre[G][NB];
#pragma unroll
    for (int p = 0; p < G; ++p) fetch(p, pre[p]);
    bool ok = true;
    const int ngrp = (nks + G - 1) / G;
    for (int g = 0; g < ngrp; ++g) {
        // the group's tile buffers are free once the previous group's MMAs are done
        if (g >= 1 && ok) ok = mbar_wait(&s_done[0], (g - 1) & 1, a.wait_us);
#pragma unroll
        for (int p = 0; p < G; ++p) {
            const int ks = g * G + p;
#pragma unroll
            for (int j = 0; j < NB; ++j) {
                const int qq = tid + kS1Threads * j;
                const int piece = qq & 7, k = (qq >> 3) & 31, bm = qq >> 8;
                const int mm = bm & 1, b = bm >> 1;
                if (ks >= nks || ks * kTcKStep + k >= n_units) continue;  // digits 0 there
                const uint32_t w[4] = {pre[p][j].x, pre[p][j].y, pre[p][j].z, pre[p][j].w};
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t lo = w[i] & 0x0F0F0F0Fu, hi = (w[i] >> 4) & 0x0F0F0F0Fu;
                    o[2 * i] = __byte_perm(lo, hi, 0x5140);      // codes of channels 8i .. 8i+3
                    o[2 * i + 1] = __byte_perm(lo, hi, 0x7362);  // channels 8i+4 .. 8i+7
                }
                const int ma = b * 2 + (piece >> 2), cc = (piece & 3) * 2;
                unsigned char *row = abuf + p * ABUF + mm * (CW * kTcKStep) + ma * LBO +
                                     (k >> 3) * 1024 + (k & 7) * 128;
                *reinterpret_cast<uint4 *>(row + (((cc) ^ (k & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4 *>(row + (((cc + 1) ^ (k & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
#pragma unroll
        for (int p = 0; p < G; ++p) fetch((g + 1) * G + p, pre[p]);
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int p = 0; p < G; ++p) {
                const int ks = g * G + p;
                if (ks >= nks) break;
                const uint32_t kb_off = (uint32_t)(ks >> 2) * (N / 8) * 1024u + (uint32_t)(ks & 3) * 32u;
#pragma unroll
                for (int mm = 0; mm < 2; ++mm) {
                    const uint64_t db = sw128_desc(baddr + mm * BM + kb_off, 16, 1024);
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
                        umma_i8(tmem + (mm * MT + mt) * N,
                                sw128_desc(aaddr + p * ABUF + mm * (CW * kTcKStep) + mt * LBO, LBO, 1024),
                                db, IDESC, ks > 0 ? 1u : 0u);
                }
            }
            // test hook: in CTA 0 this group's completion is never signalled
            if (!(a.debug_skip == g && blockIdx.x == 0)) umma_commit(&s_done[0]);
        }
    }
    if (ngrp > 0 && ok) ok = mbar_wait(&s_done[0], (ngrp - 1) & 1, a.wait_us);
    if (!ok) atomicOr(a.status, kStTimeoutMma);
    // tensor memory is read and freed only once every MMA issued has completed
    // (a wait that gave up may leave MMAs of later groups running)
    if (tid == 0) umma_commit(&s_done[1]);
    mbar_wait(&s_done[1], 0, kDefaultWaitUs);
    tc_fence_after();
    // epilogue: warp quadrant q reads TMEM lanes 32q..32q+31 (channels of an M
    // tile); the four groups of four warps take the (matrix, M tile) pairs
    const int q = wid & 3;
    for (int pi = wid >> 2; pi < 2 * MT; pi += kS1Threads / 128) {
        const int mm = pi / MT, mt = pi % MT;
        uint32_t D[N];
        if (nks > 0) {
            if constexpr (N == 32) tmem_ld32(tmem + pi * N + ((uint32_t)(q * 32) << 16), D);
            else tmem_ld16(tmem + pi * N + ((uint32_t)(q * 32) << 16), D);
        }
        const int ch = mt * 128 + q * 32 + lane;
#pragma unroll
        for (int t = 0; t < B; ++t) {
            long long V = 0;
            if (nks > 0) {
#pragma unroll
                for (int l = 0; l < 4; ++l)
                    V += ((long long)(int)D[t * 4 + l] - 8ll * s_S[mm][t][l]) * (1ll << (7 * l));
            }
            part[(mm * B + t) * CW + ch] = (float)ldexp((double)V, -(s_F[mm][t] + E[t]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (wid == 0) {
        tc_fence_after();
        tmem_free(tmem, TCOLS);
    }
}

template <int B, int NB, int PK, int TC = 0>
__global__ void __launch_bounds__(kS1Threads, 1) k_stage1(const Stage1Args a) {
    using T = S1<B, NB, PK>;
    extern __shared__ __align__(16) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    cg::cluster_group cluster = cg::this_cluster();
    const int r = (int)cluster.block_rank();  // row group
    const int c0 = (blockIdx.x / a.n_r) * NB;  // first column block of the group
    const S1Smem L = s1_smem(a.d, B, NB, a.unit_cap, a.depth_sel, kS1MaxRowGroups, PK, TC);
    unsigned char *ring = smem + L.ring;
    float *red = reinterpret_cast<float *>(smem + L.red);
    int *rowidx = reinterpret_cast<int *>(smem + L.rowidx);          // [unit_cap]
    float *xs = reinterpret_cast<float *>(smem + L.xs);              // [unit_cap][2][B]
    float *part = reinterpret_cast<float *>(smem + L.part);          // [n_r or 1][2][B][CW]
    constexpr bool kPush = (B <= 2);
    // B <= 2: each rank stores its partials straight into slot r of CTA 0's array
    float *dst_part = kPush ? cluster.map_shared_rank(part, 0) + (size_t)r * 2 * B * T::CW : part;
    __shared__ int s_warp[kS1Threads / 32];
    __shared__ __align__(16) float s_red[kS1Threads / 32][kMaxB];
    __shared__ int s_cnt[kS1Threads / 32][kMaxB + 1];
    __shared__ float s_off[T::CPT == 32 ? T::RL : 1][2][T::CPT == 32 ? B : 1];  // row-lane offset sums
    // every CTA of the cluster has started once this phase completes: only
    // then may ranks store into CTA 0's shared memory (waited for before (6))
    if (kPush) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    if (tid == 0) stamp_min(a.stamps, kS1Entry);

    // (2a) The proxy scales are layer weights, not written by the kernel
    // this launch may overlap: thread tid loads those of its K adjacent
    // 8-coordinate chunks [tid * K, tid * K + K) (K = 1, or 2 when d_model >
    // 4096) while the previous kernel of the stream finishes.
    const int NC = a.d / 8;
    const int K = (NC + kS1Threads - 1) / kS1Threads;
    float4 su[T::KMAX][2], sg[T::KMAX][2];
#pragma unroll
    for (int k = 0; k < T::KMAX; ++k) {
        const int ci = tid * K + k;
        const bool on = k < K && ci < NC;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            // a bf16 proxy has no scales: x_i enters as it is
            su[k][h] = sg[k][h] = PK ? make_float4(1.f, 1.f, 1.f, 1.f) : make_float4(0.f, 0.f, 0.f, 0.f);
            if (on && PK == 0) {
                su[k][h] = *reinterpret_cast<const float4 *>(a.s_up + ci * 8 + 4 * h);
                sg[k][h] = *reinterpret_cast<const float4 *>(a.s_gate + ci * 8 + 4 * h);
            }
        }
    }

    // Programmatic dependent launch: x, y and the workspace may belong to the
    // previous kernel in the stream; wait for it, then let the next kernel
    // (Stage 2) start its own prologue.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    if (tid == 0) {
        stamp_min(a.stamps, kS1Go);
        stamp_max(a.stamps, kS1GoMax);
    }

    // (2b) input masks m_x = 1[|x_i| >= tau_x] per token: x of the thread's
    // chunks with 16-byte loads (all issued before any use); their keep bits
    // and max |x| per token (which fixes the power-of-two pre-scale 2^E, see
    // the decode note above).
    uint4 xv[T::KMAX][B];
    uint32_t kb[T::KMAX][B];  // keep bits of the chunk per token (8 used)
#pragma unroll
    for (int k = 0; k < T::KMAX; ++k) {
        const int ci = tid * K + k;
        const bool on = k < K && ci < NC;
#pragma unroll
        for (int t = 0; t < B; ++t) {
            xv[k][t] = make_uint4(0, 0, 0, 0);
            if (on && t < a.nb) xv[k][t] = *reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.d + ci * 8);
        }
    }

    // (1) Stage 2 accumulates y with atomics: clear it here (or start it
    // from y_init, the residual stream of a layer stack), while x is on its
    // way.
    if (a.y_zero) {
        float4 *y4 = reinterpret_cast<float4 *>(a.y_zero);
        const float4 *i4 = reinterpret_cast<const float4 *>(a.y_init);
        const int n4 = a.nb * a.d / 4;
        for (int k = blockIdx.x * kS1Threads + tid; k < n4; k += gridDim.x * kS1Threads)
            y4[k] = i4 ? i4[k] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // the tensor-core Stage 2 sums split partials and counts arrivals with
    // atomics: clear them too
    if (a.z_clear)
        for (int k = blockIdx.x * kS1Threads + tid; k < a.z_n16; k += gridDim.x * kS1Threads)
            a.z_clear[k] = make_uint4(0u, 0u, 0u, 0u);

    int cnt = 0;        // union-kept coordinates of this thread
    uint32_t ub[T::KMAX];  // union keep bits per chunk
    {
        float xmax[B];
#pragma unroll
        for (int t = 0; t < B; ++t) xmax[t] = 0.f;
#pragma unroll
        for (int k = 0; k < T::KMAX; ++k) {
            const int ci = tid * K + k;
            ub[k] = 0;
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
                if (t >= a.nb || k >= K || ci >= NC) bits = 0;
                kb[k][t] = bits;
                ub[k] |= bits;
                if (a.mask_x && blockIdx.x == 0 && t < a.nb && k < K && ci < NC) {
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
            cnt += __popc(ub[k]);
        }
#pragma unroll
        for (int t = 0; t < B; ++t) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                xmax[t] = fmaxf(xmax[t], __shfl_xor_sync(0xffffffffu, xmax[t], o));
            if (lane == 0) s_red[wid][t] = xmax[t];
        }
    }

    // (3) ranks of the union-kept rows (one block-wide scan, which also
    // publishes the per-warp maxima) and this CTA's share [lo, hi) of them.
    // Each thread writes the row index and x_i * scale_i * 2^E (per matrix and
    // token; exact power-of-two scaling split in two normal-float factors) of
    // its own kept coordinates that fall in the share: no gathers.
    int kx;
    const int woffs = block_excl_scan(cnt, s_warp, kx);  // syncs the CTA
    // (kx <= 8192 and r < 8: the products fit in 32 bits)
    const int lo = kx * r / a.n_r;
    const int hi = kx * (r + 1) / a.n_r;
    const int n_units = hi - lo;
    int E[B];
#pragma unroll
    for (int t = 0; t < B; ++t) {
        // max |x| over the CTA's warps; non-negative floats order as their
        // bit patterns, and x is bf16, so a nonzero maximum is at least 2^-133
        // and ilogb is the biased exponent (normal) or the position of the top
        // mantissa bit (subnormal)
        float m4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w = 0; w < kS1Threads / 32; ++w) m4[w & 3] = fmaxf(m4[w & 3], s_red[w][t]);
        const uint32_t mb = __float_as_uint(fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
        const int be = (int)(mb >> 23);
        const int lg = be ? be - 127 : (31 - __clz((int)mb)) - 149;
        // |x * 2^E| < 2^96: a row sum of (q + 8) * x_i * scale_i * 2^E over
        // <= 8192 rows stays finite for scales below 2^15 and, for scales
        // above 2^-70, partial sums of the subnormal-coded products stay normal
        E[t] = (PK == 0 && mb != 0u) ? 95 - lg : 0;  // bf16 proxy: no pre-scale
    }
    if (woffs < hi && woffs + cnt > lo) {
        float pe1[B], pe2[B];
#pragma unroll
        for (int t = 0; t < B; ++t) {
            const int e1 = E[t] / 2, e2 = E[t] - e1;
            pe1[t] = __int_as_float((127 + e1) << 23);
            pe2[t] = __int_as_float((127 + e2) << 23);
        }
        int rank = woffs;
#pragma unroll
        for (int k = 0; k < T::KMAX; ++k) {
            if (k >= K) break;  // uniform over the grid
            const float sus[8] = {su[k][0].x, su[k][0].y, su[k][0].z, su[k][0].w,
                                  su[k][1].x, su[k][1].y, su[k][1].z, su[k][1].w};
            const float sgs[8] = {sg[k][0].x, sg[k][0].y, sg[k][0].z, sg[k][0].w,
                                  sg[k][1].x, sg[k][1].y, sg[k][1].z, sg[k][1].w};
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                if (!((ub[k] >> b) & 1u)) continue;
                if (rank >= lo && rank < hi) {
                    const int u = rank - lo;
                    rowidx[u] = (tid * K + k) * 8 + b;
#pragma unroll
                    for (int t = 0; t < B; ++t) {
                        const uint32_t w = (b & 1) ? (&xv[k][t].x)[b / 2] & 0xFFFF0000u
                                                   : (&xv[k][t].x)[b / 2] << 16;
                        const float xx = ((kb[k][t] >> b) & 1u) ? __uint_as_float(w) : 0.f;
                        xs[(u * 2 + 0) * B + t] = (xx * sus[b]) * pe1[t] * pe2[t];
                        xs[(u * 2 + 1) * B + t] = (xx * sgs[b]) * pe1[t] * pe2[t];
                    }
                }
                ++rank;
            }
        }
    }
    __syncthreads();
    if (tid == 0) stamp_max(a.stamps, kS1Pro);

    if constexpr (TC) {
        s1_tc_stream<B, NB>(a, ring, rowidx, xs, n_units, E, c0, dst_part);
        if (tid == 0) stamp_max(a.stamps, kS1Stream);
    } else {
        const int rl = tid / T::TPR;
        const int m = (tid / T::TPRM) & 1;
        const int chunk = tid % T::TPRM;
        const uint8_t *qbase = (m ? a.q_gate : a.q_up) +
                               (size_t)(c0 + chunk / T::TPRB) * a.d * T::GRAN +
                               (chunk % T::TPRB) * T::BYTES;
        const int n_rows = n_units > rl ? (n_units - rl + T::RL - 1) / T::RL : 0;
        float2 acc2[T::ACC / 2];
    #pragma unroll
        for (int k = 0; k < T::ACC / 2; ++k) acc2[k] = make_float2(0.f, 0.f);
        float ssum[B];
    #pragma unroll
        for (int t = 0; t < B; ++t) ssum[t] = 0.f;
        if (a.depth_sel == 0)
            s1_stream<B, NB, PK, T::DMAX>(qbase, ring, rowidx, xs, rl, m, n_rows, acc2, ssum);
        else if (a.depth_sel == 1)
            s1_stream<B, NB, PK, T::DMAX / 2>(qbase, ring, rowidx, xs, rl, m, n_rows, acc2, ssum);
        else
            s1_stream<B, NB, PK, T::DMAX / 4>(qbase, ring, rowidx, xs, rl, m, n_rows, acc2, ssum);
        __syncthreads();  // every thread is done with the ring before it becomes `red`
        if (tid == 0) stamp_max(a.stamps, kS1Stream);
        if (kPush) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");

        // (6) reduce row lanes, undo the pre-scale and the +8 code offset:
        // this CTA's partial sums in `part`
        if constexpr (T::CPT == 32) {
            // 32-channel chunks: 16-byte unit i of chunk c sits at unit
            // i ^ (c % 8) of the chunk (conflict-free 16-byte stores and
            // loads); each thread then sums four adjacent channels over the
            // row lanes with 16-byte loads and pushes them with one store.
            // The row lanes' offset sums go to s_off.
    #pragma unroll
            for (int t = 0; t < B; ++t) {
                float *row = red + ((size_t)((rl * 2 + m) * B + t) * T::CW) + chunk * 32;
    #pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<float4 *>(row + 4 * (i ^ (chunk & 7))) =
                        make_float4(acc2[(t * 32 + 4 * i) / 2].x, acc2[(t * 32 + 4 * i) / 2].y,
                                    acc2[(t * 32 + 4 * i) / 2 + 1].x, acc2[(t * 32 + 4 * i) / 2 + 1].y);
                if (chunk == 0) s_off[rl][m][t] = ssum[t];
            }
            __syncthreads();
            for (int o = tid; o < 2 * T::CW / 4; o += kS1Threads) {
                const int mm = o / (T::CW / 4), ch0 = (o % (T::CW / 4)) * 4;
                const int c = ch0 / 32, j = (ch0 % 32) / 4;
                const int pos = c * 32 + 4 * (j ^ (c & 7));
    #pragma unroll
                for (int t = 0; t < B; ++t) {
                    float4 sacc = make_float4(0.f, 0.f, 0.f, 0.f);
                    float soff = 0.f;
    #pragma unroll
                    for (int q = 0; q < T::RL; ++q) {
                        const float4 v = *reinterpret_cast<const float4 *>(
                            red + (size_t)((q * 2 + mm) * B + t) * T::CW + pos);
                        sacc.x += v.x; sacc.y += v.y; sacc.z += v.z; sacc.w += v.w;
                        soff += s_off[q][mm][t];
                    }
                    const int e1 = E[t] / 2, e2 = E[t] - e1;
                    const float pe = __int_as_float((127 - e1) << 23), pf = __int_as_float((127 - e2) << 23);
                    const float sv[4] = {sacc.x, sacc.y, sacc.z, sacc.w};
                    float ov[4];
    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        // 2^(149 - 4p) as a product of normal floats, p the nibble position
                        const int p = nib_pos((ch0 + e) % 8);
                        const float v = (sv[e] * __int_as_float((127 + 75) << 23)) *
                                            __int_as_float((127 + 74 - 4 * p) << 23) -
                                        8.f * soff;  // sum (q + 8 - 8) x s 2^E
                        ov[e] = v * pe * pf;
                    }
                    *reinterpret_cast<float4 *>(dst_part + (mm * B + t) * T::CW + ch0) =
                        make_float4(ov[0], ov[1], ov[2], ov[3]);
                }
            }
        } else {
        // padded rows (conflict-free both ways); the pad word after chunk 0's
        // channels carries the row lane's offset sum
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
                if constexpr (PK == 0) {
                    const int e1 = E[t] / 2, e2 = E[t] - e1;
                    const float v = (sacc * up1) * up2 - 8.f * soff;  // sum (q + 8 - 8) x s 2^E
                    dst_part[(mm * B + t) * T::CW + ch] =
                        v * __int_as_float((127 - e1) << 23) * __int_as_float((127 - e2) << 23);
                } else {
                    (void)up1, (void)up2, (void)soff;
                    dst_part[(mm * B + t) * T::CW + ch] = sacc;  // plain x_i * w_ij sums
                }
            }
        }
        }
    }
    cluster.sync();  // all partials of the block are in their CTAs' shared memory
    if (r == 0 && tid == 0) stamp_max(a.stamps, kS1Red);

    if (r == 0) {
        // (7) CTA 0 of the cluster: gather the cluster's partials (in rank
        // order), release the peers, then s~ = u~ * SiLU(g~),
        // m_s = 1[|s~| >= tau_s] and the ascending compaction per token and of
        // the union (thread = channel)
        const int ch = tid;                  // channel within the CTA's columns
        const int j = c0 * kCB + ch;         // channel index
        const int blk = wid / (kCB / 32);    // block of this warp's channels
        float uu[B], gg[B];
        // tokens in groups of up to 4: all (remote) loads of a group first,
        // then its sums in rank order
        constexpr int TG = B > 4 ? 4 : B;
#pragma unroll
        for (int t0 = 0; t0 < B; t0 += TG) {
            float pu[kS1MaxRowGroups][TG], pg[kS1MaxRowGroups][TG];
#pragma unroll
            for (int q = 0; q < kS1MaxRowGroups; ++q) {
                const float *pq = kPush ? part + (size_t)q * 2 * B * T::CW
                                        : cluster.map_shared_rank(part, q < a.n_r ? q : 0);
#pragma unroll
                for (int tt = 0; tt < TG; ++tt) {
                    pu[q][tt] = pg[q][tt] = 0.f;
                    if (q < a.n_r && t0 + tt < a.nb && ch < T::CW) {
                        pu[q][tt] = pq[(0 * B + t0 + tt) * T::CW + ch];
                        pg[q][tt] = pq[(1 * B + t0 + tt) * T::CW + ch];
                    }
                }
            }
#pragma unroll
            for (int tt = 0; tt < TG; ++tt) {
                uu[t0 + tt] = gg[t0 + tt] = 0.f;
#pragma unroll
                for (int q = 0; q < kS1MaxRowGroups; ++q) {
                    uu[t0 + tt] += pu[q][tt];
                    gg[t0 + tt] += pg[q][tt];
                }
            }
        }
        if (!kPush) asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
        uint32_t bits = 0;
#pragma unroll
        for (int t = 0; t < B; ++t) {
            if (t >= a.nb || ch >= T::CW) break;
            const float st = uu[t] * gate_act(gg[t], a.act);
            if (a.s_out) a.s_out[(size_t)t * a.f + j] = st;
            const bool keep = fabsf(st) >= a.tau_s;
            if (a.mask_s) a.mask_s[(size_t)t * a.f + j] = keep ? 1 : 0;
            bits |= (keep ? 1u : 0u) << t;
        }
        if (a.build_lists) {
            // warp ballots and per-warp counts (token t in column t, union in
            // column B). A one-token pass writes only the union list and
            // count: they are the token's (Stage 2 reads them for both).
            constexpr int T0 = B == 1 ? 1 : 0;
            uint32_t bal[kMaxB + 1];
#pragma unroll
            for (int t = T0; t <= B; ++t) {
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
                for (int t = T0; t <= B; ++t) {
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
        if (!kPush) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    } else if (!kPush) {
        // peers keep their shared memory until CTA 0 has gathered it
        asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
        asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    }
    if (a.stamps) {  // uniform over the grid
        __syncthreads();
        if (tid == 0) stamp_max(a.stamps, kS1End);
    }
}

// deepest ring that fits next to `unit_cap` rows (2 = the shallowest), or -1
int s1_depth_sel(int d, int B, int NB, int unit_cap, int PK = 0, int TC = 0) {
    for (int sel = 0; sel <= 2; ++sel)
        if (s1_smem(d, B, NB, unit_cap, sel, kS1MaxRowGroups, PK, TC).total <= (size_t)kS2SmemBudget)
            return sel;
    return -1;
}

template <int B, int NB, int PK, int TC = 0>
cudaError_t launch1(Stage1Args a, const Stage1Plan &p0, cudaStream_t s) {
    auto k = k_stage1<B, NB, PK, TC>;
    const int groups = a.C / NB;  // clusters
    // Cluster size (row groups per block): every cluster of the grid must be
    // resident at once, or the last clusters run as a second wave. Start from
    // the plan's choice and shrink until the occupancy calculator agrees.
    // (per device: the shared-memory attribute and the occupancy are per device)
    struct Cache {
        int d = 0, C = 0, n_r = 0, cap = 0, sel = 0;
        size_t smem = 0;
    };
    static Cache caches[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::unique_lock<std::mutex> lk(mu);
    Cache &cache = caches[dev];
    Stage1Plan p = p0;
    if (cache.d == a.d && cache.C == a.C) {
        p.n_r = cache.n_r;
        p.unit_cap = cache.cap;
        p.depth_sel = cache.sel;
        p.smem = cache.smem;
    } else {
        // fewest row groups whose rows fit in one CTA's shared memory
        int n_min = 1;
        while (n_min < kS1MaxRowGroups &&
               s1_depth_sel(a.d, B, NB, (a.d + n_min - 1) / n_min, PK, TC) < 0)
            ++n_min;
        if (p.n_r < n_min) p.n_r = n_min;
        for (;;) {
            p.unit_cap = (a.d + p.n_r - 1) / p.n_r;
            p.depth_sel = s1_depth_sel(a.d, B, NB, p.unit_cap, PK, TC);
            if (p.depth_sel < 0) return cudaErrorInvalidConfiguration;
            p.smem = s1_smem(a.d, B, NB, p.unit_cap, p.depth_sel, kS1MaxRowGroups, PK, TC).total;
            cudaError_t e = set_max_dynamic_smem((const void *)k, p.smem);
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
        cache.sel = p.depth_sel;
        cache.smem = p.smem;
    }
    lk.unlock();
    a.n_r = p.n_r;
    a.unit_cap = p.unit_cap;
    a.depth_sel = p.depth_sel;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(groups * a.n_r);
    cfg.blockDim = dim3(kS1Threads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    // Load-balancing cluster placement: with the default policy the clusters
    // of some processes are placed late while the previous kernel's CTAs
    // leave their SMs, and the first and last CTA pass the grid wait about
    // 1 us apart (0.06 us with this policy, every run measured).
    cudaLaunchAttribute attr[3];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = a.n_r;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    attr[2].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[2].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicyLoadBalancing;
    cfg.attrs = attr;
    cfg.numAttrs = 3;
    return cudaLaunchKernelEx(&cfg, k, a);
}

}  // namespace

cudaError_t launch_stage1(int B, const Stage1Args &a, const Stage1Plan &p, cudaStream_t s) {
#define PROX_S1(BB, NN)                                                          \
    if (B == BB && p.nb_blocks == NN)                                            \
        return a.pk ? launch1<BB, NN, 1>(a, p, s) : launch1<BB, NN, 0>(a, p, s);
    // the tensor-core stream: passes of 4 or 8 tokens, INT4 proxy. Over
    // one-block columns it is the only stream for such passes: the CUDA-core
    // stream of 4 tokens over one-block columns of a 4096-wide layer stopped
    // with an illegal-instruction error once, for a reason not yet found, so
    // that configuration is never launched.
    if (a.pk == 0 && (B == 4 || B == 8) && (a.tc || p.nb_blocks == 1)) {
        if (B == 4) return p.nb_blocks == 2 ? launch1<4, 2, 0, 1>(a, p, s) : launch1<4, 1, 0, 1>(a, p, s);
        return p.nb_blocks == 2 ? launch1<8, 2, 0, 1>(a, p, s) : launch1<8, 1, 0, 1>(a, p, s);
    }
    PROX_S1(1, 1) PROX_S1(1, 2) PROX_S1(2, 1) PROX_S1(2, 2)
    PROX_S1(4, 1) PROX_S1(4, 2) PROX_S1(8, 1) PROX_S1(8, 2)
#undef PROX_S1
    return cudaErrorInvalidValue;
}

size_t stage1_smem_bytes(int d_model, int B, int NB, int unit_cap) {
    const int sel = s1_depth_sel(d_model, B, NB, unit_cap);
    return s1_smem(d_model, B, NB, unit_cap, sel < 0 ? 2 : sel).total;
}

}  // namespace prox
