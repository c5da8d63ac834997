// Offline kernels: symmetric per-row INT4 proxy quantisation (Prox deep-dive
// blog, section "Stage 1": W~_up and W~_gate are symmetric per-row INT4
// copies) and the exact order statistics used for threshold calibration
// (blog, "Stage 1" and "Evidence": per-layer thresholds from calibration
// activations).
//
// Quantisation, per row i of W in the pages' orientation (d_model x d_ff),
// i.e. per column i of the channel-major weight:
//   scale_i = RN(max_j |W[i,j]| / 7),  q_ij = clamp(RN_even(RN(W[i,j] / scale_i)), -7, 7)
// with IEEE fp32 division (__fdiv_rn) and round-half-even (__float2int_rn);
// an all-zero row gives scale 0 and q 0. Packing (block-tiled, the layout
// Stage 1 streams): byte m of granule q[c][i] holds channel 256c + 2m in the
// low nibble and 256c + 2m + 1 in the high nibble, each stored offset-binary
// as q + 8 (1..15), which is the form Stage 1's decode consumes directly.
//
// Order statistic: the magnitude bit patterns of non-negative IEEE numbers
// sort like unsigned integers, so the rank-k magnitude is found exactly by
// histogram radix selection (one 15-bit pass for bf16, a 16-bit and a 15-bit
// pass for fp32) with no sort and no rounding.
#include "prox_internal.cuh"

#include <cuda_runtime.h>
#include <cstdint>

namespace prox {
namespace {

constexpr int kQRows = 32;    // input rows (columns of w_cm) per CTA
constexpr int kQChan = 256;   // channels per CTA in the packing kernel

__global__ void __launch_bounds__(256) k_colmax(int d, int f, const uint16_t *__restrict__ w,
                                                float *__restrict__ scale) {
    __shared__ float sm[8][kQRows];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int i = blockIdx.x * kQRows + lane;
    float m = 0.f;
    for (int j = wid; j < f; j += 8)
        m = fmaxf(m, fabsf(__uint_as_float((uint32_t)w[(size_t)j * d + i] << 16)));
    sm[wid][lane] = m;
    __syncthreads();
    if (wid == 0) {
#pragma unroll
        for (int k = 1; k < 8; ++k) m = fmaxf(m, sm[k][lane]);
        scale[i] = __fdiv_rn(m, 7.0f);
    }
}

__global__ void __launch_bounds__(256) k_pack(int d, int f, const uint16_t *__restrict__ w,
                                              const float *__restrict__ scale,
                                              uint8_t *__restrict__ q) {
    __shared__ uint16_t tile[kQChan][kQRows + 2];
    const int i0 = blockIdx.x * kQRows, j0 = blockIdx.y * kQChan;
    for (int k = threadIdx.x; k < kQChan * kQRows; k += 256) {
        const int jj = k / kQRows, ii = k % kQRows;
        tile[jj][ii] = w[(size_t)(j0 + jj) * d + i0 + ii];
    }
    __syncthreads();
    const int ii = threadIdx.x / 8, chunk = threadIdx.x % 8;  // 32 channels per thread
    const float s = scale[i0 + ii];
    uint32_t out[4] = {0, 0, 0, 0};
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float wv = __uint_as_float((uint32_t)tile[chunk * 32 + k][ii] << 16);
        int v = 0;
        if (s > 0.f) {
            v = __float2int_rn(__fdiv_rn(wv, s));
            v = v > 7 ? 7 : (v < -7 ? -7 : v);
        }
        out[k / 8] |= (uint32_t)(v + 8) << (4 * (k % 8));
    }
    // block-tiled output: q[c][i][0..127] holds channels [256c, 256c + 256) of row i
    const int cblk = j0 / kCB, mbyte = (j0 % kCB + chunk * 32) / 2;
    *reinterpret_cast<uint4 *>(q + ((size_t)cblk * d + i0 + ii) * (kCB / 2) + mbyte) =
        make_uint4(out[0], out[1], out[2], out[3]);
}

// bf16 proxy tiles: q16[(c * d + i) * 256 + k] = w[(256 c + k) * d + i], a
// tiled transpose through shared memory (32 rows x 256 channels per CTA)
__global__ void __launch_bounds__(256) k_tile_bf16(int d, const uint16_t *__restrict__ w,
                                                   uint16_t *__restrict__ q16) {
    __shared__ uint16_t tile[kQChan][kQRows + 2];
    const int i0 = blockIdx.x * kQRows, c = blockIdx.y;
    for (int k = threadIdx.x; k < kQChan * kQRows; k += 256) {
        const int jj = k / kQRows, ii = k % kQRows;
        tile[jj][ii] = w[(size_t)(c * kCB + jj) * d + i0 + ii];
    }
    __syncthreads();
    for (int k = threadIdx.x; k < kQChan * kQRows; k += 256) {
        const int ii = k / kQChan, jj = k % kQChan;
        q16[((size_t)c * d + i0 + ii) * kCB + jj] = tile[jj][ii];
    }
}

__global__ void k_hist_bf16_abs(const uint16_t *__restrict__ v, long n, uint32_t *hist) {
    for (long k = blockIdx.x * (long)blockDim.x + threadIdx.x; k < n;
         k += (long)gridDim.x * blockDim.x)
        atomicAdd(&hist[v[k] & 0x7FFFu], 1u);
}

__global__ void k_hist_f32_hi(const float *__restrict__ v, long n, uint32_t *hist) {
    for (long k = blockIdx.x * (long)blockDim.x + threadIdx.x; k < n;
         k += (long)gridDim.x * blockDim.x)
        atomicAdd(&hist[(__float_as_uint(v[k]) & 0x7FFFFFFFu) >> 15], 1u);
}

__global__ void k_hist_f32_lo(const float *__restrict__ v, long n, const uint32_t *sel,
                              uint32_t *hist) {
    const uint32_t hb = sel[0];
    for (long k = blockIdx.x * (long)blockDim.x + threadIdx.x; k < n;
         k += (long)gridDim.x * blockDim.x) {
        const uint32_t b = __float_as_uint(v[k]) & 0x7FFFFFFFu;
        if ((b >> 15) == hb) atomicAdd(&hist[b & 0x7FFFu], 1u);
    }
}

// One CTA of 1024 threads: the bin holding rank `rank` (or *rank_io when
// given); writes the bin to sel[slot] and the rank left inside it to *rank_io.
__global__ void __launch_bounds__(1024) k_select(const uint32_t *hist, int nbins, long long rank,
                                                 long long *rank_io, uint32_t *sel, int slot) {
    __shared__ long long wsum[32];
    __shared__ long long s_rank;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) s_rank = rank_io && slot > 0 ? *rank_io : rank;
    const int per = nbins / 1024;
    long long loc = 0;
    for (int k = 0; k < per; ++k) loc += hist[tid * per + k];
    long long inc = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long nb = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += nb;
    }
    if (lane == 31) wsum[wid] = inc;
    __syncthreads();
    long long base = 0;
    for (int w = 0; w < wid; ++w) base += wsum[w];
    long long cum = base + inc - loc;  // count of values in bins before this thread's
    const long long r = s_rank;
    if (r >= cum && r < cum + loc) {
        for (int k = 0; k < per; ++k) {
            const long long h = hist[tid * per + k];
            if (r < cum + h) {
                sel[slot] = (uint32_t)(tid * per + k);
                if (rank_io) *rank_io = r - cum;
                break;
            }
            cum += h;
        }
    }
}

__global__ void k_tau_bf16(const uint32_t *sel, float *tau) { *tau = __uint_as_float(sel[0] << 16); }

// Histogram quantile (every k-th of n values, `bins` equal bins over [0, m],
// m the largest sample; tau = the lower edge of the bin holding the rank-r
// sample): fp32 magnitude of value i, for bf16 or fp32 inputs
template <typename V>
__device__ __forceinline__ float mag(const V *v, long i);
template <>
__device__ __forceinline__ float mag<uint16_t>(const uint16_t *v, long i) {
    return __uint_as_float((uint32_t)(v[i] & 0x7FFFu) << 16);
}
template <>
__device__ __forceinline__ float mag<float>(const float *v, long i) {
    return fabsf(v[i]);
}

// scratch[2] = bit pattern of the largest sample (non-negative floats order
// like their bit patterns)
template <typename V>
__global__ void k_sub_max(const V *__restrict__ v, long ns, long k, uint32_t *scratch) {
    uint32_t m = 0;
    for (long s = blockIdx.x * (long)blockDim.x + threadIdx.x; s < ns;
         s += (long)gridDim.x * blockDim.x)
        m = max(m, __float_as_uint(mag(v, s * k)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(&scratch[2], m);
}

template <typename V>
__global__ void k_sub_hist(const V *__restrict__ v, long ns, long k, int bins,
                           const uint32_t *scratch, uint32_t *hist) {
    const float m = __uint_as_float(scratch[2]);
    if (m == 0.f) return;
    const float w = __fdiv_rn(m, (float)bins);
    for (long s = blockIdx.x * (long)blockDim.x + threadIdx.x; s < ns;
         s += (long)gridDim.x * blockDim.x) {
        const float q = __fdiv_rn(mag(v, s * k), w);
        int b = (int)q;  // q >= 0: truncation
        if (b > bins - 1) b = bins - 1;
        atomicAdd(&hist[b], 1u);
    }
}

__global__ void k_tau_hist(const uint32_t *scratch, int bins, float *tau) {
    const float m = __uint_as_float(scratch[2]);
    *tau = (m == 0.f) ? 0.f : (float)scratch[0] * __fdiv_rn(m, (float)bins);
}
__global__ void k_tau_f32(const uint32_t *sel, float *tau) {
    *tau = __uint_as_float((sel[0] << 15) | sel[1]);
}

}  // namespace

cudaError_t launch_tile_bf16(int d, int f, const uint16_t *w_cm, uint16_t *q16, cudaStream_t s) {
    k_tile_bf16<<<dim3(d / kQRows, f / kCB), 256, 0, s>>>(d, w_cm, q16);
    return cudaGetLastError();
}

cudaError_t launch_quantize(int d, int f, const uint16_t *w_cm, uint8_t *q, float *scale,
                            cudaStream_t s) {
    k_colmax<<<d / kQRows, 256, 0, s>>>(d, f, w_cm, scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_pack<<<dim3(d / kQRows, f / kQChan), 256, 0, s>>>(d, f, w_cm, scale, q);
    return cudaGetLastError();
}

// Histogram threshold of |v| (bf16 bit patterns or fp32): ns = ceil(n / k)
// samples v[0], v[k], ...; rank counts within the samples; bins a multiple of
// 1024, at most 65536. scratch: >= 16 bytes; hist: `bins` words.
template <typename V>
cudaError_t launch_hist_quantile(const V *v, long n, long k, long rank, int bins, uint32_t *hist,
                                 uint32_t *scratch, float *tau_dev, cudaStream_t s) {
    const long ns = (n + k - 1) / k;
    cudaError_t e = cudaMemsetAsync(hist, 0, (size_t)bins * sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(scratch, 0, 3 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    k_sub_max<V><<<1184, 256, 0, s>>>(v, ns, k, scratch);
    k_sub_hist<V><<<1184, 256, 0, s>>>(v, ns, k, bins, scratch, hist);
    k_select<<<1, 1024, 0, s>>>(hist, bins, rank, nullptr, scratch, 0);
    k_tau_hist<<<1, 1, 0, s>>>(scratch, bins, tau_dev);
    return cudaGetLastError();
}

cudaError_t launch_hist_quantile_bf16(const uint16_t *v, long n, long k, long rank, int bins,
                                      uint32_t *hist, uint32_t *scratch, float *tau_dev,
                                      cudaStream_t s) {
    return launch_hist_quantile(v, n, k, rank, bins, hist, scratch, tau_dev, s);
}
cudaError_t launch_hist_quantile_f32(const float *v, long n, long k, long rank, int bins,
                                     uint32_t *hist, uint32_t *scratch, float *tau_dev,
                                     cudaStream_t s) {
    return launch_hist_quantile(v, n, k, rank, bins, hist, scratch, tau_dev, s);
}

// scratch: >= 16 bytes (two selected bins) + 8 bytes (rank); hist: 65536 words
cudaError_t launch_select_bf16_abs(const uint16_t *v, long n, long rank, uint32_t *hist,
                                   uint32_t *scratch, float *tau_dev, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(hist, 0, 32768 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    k_hist_bf16_abs<<<1184, 256, 0, s>>>(v, n, hist);
    k_select<<<1, 1024, 0, s>>>(hist, 32768, rank, nullptr, scratch, 0);
    k_tau_bf16<<<1, 1, 0, s>>>(scratch, tau_dev);
    return cudaGetLastError();
}

cudaError_t launch_select_f32_abs(const float *v, long n, long rank, uint32_t *hist,
                                  uint32_t *scratch, float *tau_dev, cudaStream_t s) {
    long long *rank_io = reinterpret_cast<long long *>(scratch + 2);
    cudaError_t e = cudaMemsetAsync(hist, 0, 65536 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    k_hist_f32_hi<<<1184, 256, 0, s>>>(v, n, hist);
    k_select<<<1, 1024, 0, s>>>(hist, 65536, rank, rank_io, scratch, 0);
    e = cudaMemsetAsync(hist, 0, 32768 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    k_hist_f32_lo<<<1184, 256, 0, s>>>(v, n, scratch, hist);
    k_select<<<1, 1024, 0, s>>>(hist, 32768, 0, rank_io, scratch, 1);
    k_tau_f32<<<1, 1, 0, s>>>(scratch, tau_dev);
    return cudaGetLastError();
}

}  // namespace prox
