// FP8 side of the 2:4 prefill (2:4 + Squared-ReLU page, 利用2:4稀疏性与
// Squared-ReLU加速Transformer训练与推理, section 3.1: one fused kernel applies
// Squared-ReLU, the 2:4 selection and FP8 quantisation to the layer input,
// and the 2:4 GEMM takes FP8 operands with row scaling; section 5.3: sparsify
// before quantising).
//
// Format: E4M3 ("fn": largest finite 448, no infinities), round to nearest
// even, saturating.  One float32 scale per row: scale = fl32(amax / 448) over
// the row's kept values, codes E4M3(fl32(v * inv)) with inv = fl32(448 / amax)
// (scale = inv = 1 for an all-zero row).
//
// k_sqrelu24_fp8     one CTA per token row: x = fl32(max(0, z))^2 from the
//                    bf16 pre-activation, 2:4 by magnitude (ties to the lower
//                    index), the row amax, then the kept values' codes, their
//                    positions in the FP8 sparse-MMA metadata layout and the
//                    optional bitmask.  x is never written; rows up to 16384
//                    channels are read once and held in registers.
// k_quant_rows_fp8   one CTA per weight row: amax, then codes.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.cuh"
#include "select_util.cuh"

namespace as {

constexpr int F8_THREADS = 256;
constexpr uint8_t F8_PAD_META = 0x44;  // positions (0, 1) in both 4-blocks of a byte

__device__ __forceinline__ float block_max(float v, float *red)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float m = red[0];
#pragma unroll
    for (int w = 1; w < F8_THREADS / 32; ++w) m = fmaxf(m, red[w]);
    return m;
}

// Eight consecutive bf16 pre-activations -> x = max(0, z)^2 in float32.
__device__ __forceinline__ void sqrelu8(const uint4 u, float (&x)[8])
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
        const float rl = lo > 0.0f ? lo : 0.0f, rh = hi > 0.0f ? hi : 0.0f;
        x[2 * i] = __fmul_rn(rl, rl);
        x[2 * i + 1] = __fmul_rn(rh, rh);
    }
}

// Byte offset of the positions of channels [8c, 8c+8) of token t in the FP8
// metadata buffer.  Tiles of 128 tokens x 256 channels, 4 KB each, tile
// (r, ct) at byte (r * kt + ct) * 4096; inside, two 2 KB halves (channels
// 0..127 and 128..255 of the tile); in a half, 16 bytes per token (its TMEM
// lane), word j%4 holding channels 32j..32j+31, 4 bits per 4-block at bit
// 4 * ((channel % 32) / 4): one byte per 8 channels.
__device__ __forceinline__ size_t meta8_byte(int t, int c, int kt)
{
    const int r = t >> 7, p = t & 127;
    const int ch = 8 * c, ct = ch >> 8, q = ch & 255, j = q >> 5;
    const size_t word = ((size_t)r * kt + ct) * 1024 + (size_t)(j >> 2) * 512 + (size_t)p * 4 + (j & 3);
    return word * 4 + (c & 3);
}

// E4M3 codes of two values, a in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b)
{
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

// Codes (4 bytes, channel order) and positions (one byte) of the kept values
// of one 8-channel chunk (two 4-blocks); `keep` gets the 8 keep bits.
__device__ __forceinline__ void chunk_codes(const float (&x)[8], float inv, uint32_t &codes, uint32_t &meta,
                                            uint32_t &keep)
{
    keep = keep_2of4<float>(x);
    const uint32_t lo = e4m3x2(__fmul_rn(x[0], inv), __fmul_rn(x[1], inv)) |
                            (e4m3x2(__fmul_rn(x[2], inv), __fmul_rn(x[3], inv)) << 16);
    const uint32_t hi = e4m3x2(__fmul_rn(x[4], inv), __fmul_rn(x[5], inv)) |
                            (e4m3x2(__fmul_rn(x[6], inv), __fmul_rn(x[7], inv)) << 16);
    int a0, a1, b0, b1;
    pos_2of4(keep & 15u, a0, a1);
    pos_2of4((keep >> 4) & 15u, b0, b1);
    // byte permutes: bytes a0, a1 of lo, then bytes b0, b1 of hi (selector 4..7)
    codes = __byte_perm(lo, hi, (uint32_t)a0 | ((uint32_t)a1 << 4) | ((uint32_t)(b0 + 4) << 8) |
                                    ((uint32_t)(b1 + 4) << 12));
    meta = (uint32_t)(a0 | (a1 << 2)) | ((uint32_t)(b0 | (b1 << 2)) << 4);
}

// Largest of eight bf16 values (as float32).
__device__ __forceinline__ float max8_bf16(const uint4 u)
{
    __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
    a = __hmax2(a, *reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    a = __hmax2(a, *reinterpret_cast<const __nv_bfloat162 *>(&u.z));
    a = __hmax2(a, *reinterpret_cast<const __nv_bfloat162 *>(&u.w));
    return fmaxf(__low2float(a), __high2float(a));
}

// A row of up to F8_HELD * 8 * F8_THREADS channels is loaded once, with all
// of a thread's loads in flight together, and kept in registers between the
// amax pass and the code pass; longer rows are processed in slices of that
// size and read again (from L2) for the codes.
constexpr int F8_HELD = 8;

// The amax over the kept values equals the amax over all of x: the largest
// value of every 4-block is among its two kept ones.  x = r * r is exact for
// a bf16 r (at most 16 significant bits) and increasing in r >= 0, so the
// amax is the square of the largest positive z.
__global__ void __launch_bounds__(F8_THREADS) k_sqrelu24_fp8(const __nv_bfloat16 *__restrict__ z, int T, int K,
                                                             uint8_t *__restrict__ x8, uint8_t *__restrict__ meta8,
                                                             float *__restrict__ x_scale,
                                                             uint8_t *__restrict__ bitmask, int kt)
{
    __shared__ float red[F8_THREADS / 32];
    const int t = blockIdx.x;
    const int nch = K / 8;          // real 8-channel chunks
    const int nch_pad = kt * 32;    // chunks the metadata tiles cover
    const int tid = threadIdx.x;
    const long long meta_bytes = (long long)((T + 255) / 256) * 2 * kt * 1024 * 4;
    for (int c = nch + tid; c < nch_pad; c += F8_THREADS)
        if (as_in((long long)meta8_byte(t, c, kt), meta_bytes)) meta8[meta8_byte(t, c, kt)] = F8_PAD_META;
    if (t >= T) {                   // padding rows of the last 256-row pair tile
        for (int c = tid; c < nch; c += F8_THREADS)
            if (as_in((long long)meta8_byte(t, c, kt), meta_bytes)) meta8[meta8_byte(t, c, kt)] = F8_PAD_META;
        return;
    }
    const __nv_bfloat16 *zr = z + (size_t)t * K;
    constexpr int SLICE = F8_HELD * F8_THREADS;  // chunks per slice
    uint4 held[F8_HELD];
    float zmax = 0.0f;
    for (int base = 0; base < nch; base += SLICE) {
#pragma unroll
        for (int r = 0; r < F8_HELD; ++r) {
            const int c = base + tid + r * F8_THREADS;
            held[r] = c < nch ? *reinterpret_cast<const uint4 *>(zr + 8 * c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int r = 0; r < F8_HELD; ++r) zmax = fmaxf(zmax, max8_bf16(held[r]));
    }
    zmax = block_max(zmax, red);
    const float amax = __fmul_rn(zmax, zmax);
    const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 1.0f;
    if (tid == 0) x_scale[t] = scale;

    uint8_t *xr = x8 + (size_t)t * (K / 2);
    const size_t bm_row = (size_t)t * ((K + 31) / 32) * 4;
    for (int base = 0; base < nch; base += SLICE) {
        if (nch > SLICE) {  // several slices: `held` has the last one, read each again
#pragma unroll
            for (int r = 0; r < F8_HELD; ++r) {
                const int c = base + tid + r * F8_THREADS;
                held[r] = c < nch ? *reinterpret_cast<const uint4 *>(zr + 8 * c) : make_uint4(0, 0, 0, 0);
            }
        }
        // chunks c and c + F8_THREADS lie 8 metadata tiles (32 KB) apart
        const size_t mb0 = meta8_byte(t, base + tid, kt);
#pragma unroll
        for (int r = 0; r < F8_HELD; ++r) {
            const int c = base + tid + r * F8_THREADS;
            if (c >= nch) break;
            float x[8];
            sqrelu8(held[r], x);
            uint32_t codes, meta, keep;
            chunk_codes(x, inv, codes, meta, keep);
            if (!as_in((long long)t * (K / 2) + 4 * c + 3, (long long)T * (K / 2)) ||
                !as_in((long long)(mb0 + (size_t)r * (F8_THREADS / 32) * 4096), meta_bytes))
                continue;
            *reinterpret_cast<uint32_t *>(xr + 4 * c) = codes;
            meta8[mb0 + (size_t)r * (F8_THREADS / 32) * 4096] = (uint8_t)meta;
            if (bitmask) bitmask[bm_row + c] = (uint8_t)keep;
        }
    }
}

template <typename TW>
__device__ __forceinline__ void load8(const TW *p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8])
{
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
template <>
__device__ __forceinline__ void load8<float>(const float *p, float (&v)[8])
{
    const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename TW>
__global__ void __launch_bounds__(F8_THREADS) k_quant_rows_fp8(const TW *__restrict__ W, int K,
                                                               uint8_t *__restrict__ Wq, float *__restrict__ w_scale)
{
    __shared__ float red[F8_THREADS / 32];
    const int o = blockIdx.x;
    const TW *wr = W + (size_t)o * K;
    const int nch = K / 8;
    float amax = 0.0f;
    for (int c = threadIdx.x; c < nch; c += F8_THREADS) {
        float v[8];
        load8<TW>(wr + 8 * c, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
    }
    amax = block_max(amax, red);
    const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 1.0f;
    if (threadIdx.x == 0) w_scale[o] = scale;
    uint8_t *qr = Wq + (size_t)o * K;
    for (int c = threadIdx.x; c < nch; c += F8_THREADS) {
        float v[8];
        load8<TW>(wr + 8 * c, v);
        const uint32_t lo = e4m3x2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv)) |
                                (e4m3x2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv)) << 16);
        const uint32_t hi = e4m3x2(__fmul_rn(v[4], inv), __fmul_rn(v[5], inv)) |
                                (e4m3x2(__fmul_rn(v[6], inv), __fmul_rn(v[7], inv)) << 16);
        *reinterpret_cast<uint2 *>(qr + 8 * c) = make_uint2(lo, hi);
    }
}

int meta8_kt(int K) { return (K + 255) / 256; }

size_t meta8_words(int T, int K) { return (size_t)((T + 255) / 256) * 2 * (size_t)meta8_kt(K) * 1024; }

cudaError_t launch_sqrelu24_fp8(const void *z, int T, int K, uint8_t *x8, uint32_t *meta8, float *x_scale,
                                uint32_t *bitmask, cudaStream_t st)
{
    const int rows_pad = (T + 255) / 256 * 256;
    k_sqrelu24_fp8<<<rows_pad, F8_THREADS, 0, st>>>(static_cast<const __nv_bfloat16 *>(z), T, K, x8,
                                                    reinterpret_cast<uint8_t *>(meta8), x_scale,
                                                    reinterpret_cast<uint8_t *>(bitmask), meta8_kt(K));
    return cudaGetLastError();
}

cudaError_t launch_quant_rows_fp8(const void *W, int bf16, int n_out, int K, uint8_t *Wq, float *w_scale,
                                  cudaStream_t st)
{
    if (bf16)
        k_quant_rows_fp8<__nv_bfloat16><<<n_out, F8_THREADS, 0, st>>>(static_cast<const __nv_bfloat16 *>(W), K, Wq,
                                                                      w_scale);
    else
        k_quant_rows_fp8<float><<<n_out, F8_THREADS, 0, st>>>(static_cast<const float *>(W), K, Wq, w_scale);
    return cudaGetLastError();
}

}  // namespace as
