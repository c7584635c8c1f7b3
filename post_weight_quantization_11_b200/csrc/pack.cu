// INT4 packing -- "INT4/INT8 量化推理" sec. 一: 128 x 4 bit = 64 B of codes,
// one 4-bit zero point (0.5 B) and one fp16 scale (2 B) per 128 weights.
// Layout: eight codes per little-endian uint32, lowest column in the lowest
// nibble; zero points two per byte, even group in the low nibble.
// Each thread produces 16 bytes of output (four uint32 words from 32 codes),
// so loads and stores are 16-byte vectors and fully coalesced.
#include "common.cuh"

namespace gptq {

__device__ __forceinline__ uint32_t pack8(uint2 c)
{
    // c.x holds codes 0..3 (one per byte), c.y codes 4..7
    uint32_t a = c.x, b = c.y;
    uint32_t lo = (a & 0xfu) | ((a >> 4) & 0xf0u) | ((a >> 8) & 0xf00u) | ((a >> 12) & 0xf000u);
    uint32_t hi = (b & 0xfu) | ((b >> 4) & 0xf0u) | ((b >> 8) & 0xf00u) | ((b >> 12) & 0xf000u);
    return lo | (hi << 16);
}

__global__ void pack_codes_kernel(const uint8_t* __restrict__ codes, int64_t total_words4,
                                  int64_t words_per_row, uint32_t* __restrict__ qweight)
{
    // one thread: 4 words (32 codes) when the row has them, else single words
    for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < total_words4;
         t += int64_t(gridDim.x) * blockDim.x) {
        const uint4* src = reinterpret_cast<const uint4*>(codes) + 2 * t;
        uint4 a = src[0], b = src[1];
        uint4 o;
        o.x = pack8(make_uint2(a.x, a.y));
        o.y = pack8(make_uint2(a.z, a.w));
        o.z = pack8(make_uint2(b.x, b.y));
        o.w = pack8(make_uint2(b.z, b.w));
        reinterpret_cast<uint4*>(qweight)[t] = o;
    }
}

__global__ void pack_codes_tail_kernel(const uint8_t* __restrict__ codes, int64_t words,
                                       uint32_t* __restrict__ qweight)
{
    for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < words;
         t += int64_t(gridDim.x) * blockDim.x) {
        const uint2 c = reinterpret_cast<const uint2*>(codes)[t];
        qweight[t] = pack8(c);
    }
}

__global__ void pack_zeros_kernel(const uint8_t* __restrict__ zeros, int64_t m, int64_t G,
                                  uint8_t* __restrict__ qzeros)
{
    const int64_t Gb = (G + 1) / 2;
    for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < m * Gb;
         t += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = t / Gb, b = t - r * Gb;
        const uint8_t lo = zeros[r * G + 2 * b] & 0xfu;
        const uint8_t hi = (2 * b + 1 < G) ? (zeros[r * G + 2 * b + 1] & 0xfu) : 0u;
        qzeros[t] = uint8_t(lo | (hi << 4));
    }
}

__global__ void unpack_codes_kernel(const uint32_t* __restrict__ qweight, int64_t words,
                                    uint8_t* __restrict__ codes)
{
    for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < words;
         t += int64_t(gridDim.x) * blockDim.x) {
        const uint32_t v = qweight[t];
        uint2 o;
        o.x = (v & 0xfu) | ((v << 4) & 0xf00u) | ((v << 8) & 0xf0000u) | ((v << 12) & 0xf000000u);
        const uint32_t u = v >> 16;
        o.y = (u & 0xfu) | ((u << 4) & 0xf00u) | ((u << 8) & 0xf0000u) | ((u << 12) & 0xf000000u);
        reinterpret_cast<uint2*>(codes)[t] = o;
    }
}

__global__ void unpack_zeros_kernel(const uint8_t* __restrict__ qzeros, int64_t m, int64_t G,
                                    uint8_t* __restrict__ zeros)
{
    const int64_t Gb = (G + 1) / 2;
    for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < m * G;
         t += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = t / G, g = t - r * G;
        const uint8_t b = qzeros[r * Gb + g / 2];
        zeros[t] = (g & 1) ? uint8_t(b >> 4) : uint8_t(b & 0xfu);
    }
}

static unsigned grid_for(int64_t n, int threads)
{
    return (unsigned)std::max<int64_t>(1, std::min<int64_t>(ceil_div(n, threads), 148 * 32));
}

// b-bit storage for the other widths (b = 2..8): each row's codes form one
// little-endian bit stream, code k in bits [b k, b k + b), stored as uint32
// words; b = 4 is the INT4 layout above.  One thread per 32-code chunk of a
// row: two 16-byte loads of codes, b words out (32 codes = 32 b bits).
template <int B>
__global__ void pack_bits_kernel(const uint8_t* __restrict__ codes, int64_t chunks,
                                 uint32_t* __restrict__ qweight)
{
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < chunks;
         i += int64_t(gridDim.x) * blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(codes + 32 * i);
    const uint4 v0 = src[0], v1 = src[1];
    const uint32_t c4[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t wd[B];
#pragma unroll
    for (int t = 0; t < B; ++t) wd[t] = 0u;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const uint32_t c = (c4[k >> 2] >> (8 * (k & 3))) & ((1u << B) - 1u);
        const int bit = B * k, w = bit >> 5, sh = bit & 31;
        wd[w] |= c << sh;
        if (sh + B > 32) wd[w + 1] |= c >> (32 - sh);
    }
    uint32_t* dst = qweight + int64_t(B) * i;
#pragma unroll
    for (int t = 0; t < B; ++t) dst[t] = wd[t];
    }
}

template <int B>
__global__ void unpack_bits_kernel(const uint32_t* __restrict__ qweight, int64_t chunks,
                                   uint8_t* __restrict__ codes)
{
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < chunks;
         i += int64_t(gridDim.x) * blockDim.x) {
    uint32_t wd[B + 1];
#pragma unroll
    for (int t = 0; t < B; ++t) wd[t] = qweight[int64_t(B) * i + t];
    wd[B] = 0u;
    uint32_t c4[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) c4[q] = 0u;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const int bit = B * k, w = bit >> 5, sh = bit & 31;
        uint32_t c = wd[w] >> sh;
        if (sh + B > 32) c |= wd[w + 1] << (32 - sh);
        c4[k >> 2] |= (c & ((1u << B) - 1u)) << (8 * (k & 3));
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + 32 * i);
    dst[0] = make_uint4(c4[0], c4[1], c4[2], c4[3]);
    dst[1] = make_uint4(c4[4], c4[5], c4[6], c4[7]);
    }
}

// Zero points: the row's stream of G b-bit values in ceil(G b / 8) bytes;
// one thread per output byte (pack) or per zero point (unpack).
__global__ void pack_zero_bits_kernel(const uint8_t* __restrict__ zeros, int64_t m, int64_t G,
                                      int b, uint8_t* __restrict__ qzeros)
{
    const int64_t nb = (G * b + 7) / 8;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < m * nb;
         i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / nb, byte = i - r * nb;
    uint32_t v = 0u;
    for (int64_t g = (8 * byte) / b; g < G && g * b < 8 * byte + 8; ++g) {
        const uint32_t z = zeros[r * G + g] & ((1u << b) - 1u);
        const int64_t sh = g * b - 8 * byte;           // may be negative
        v |= sh >= 0 ? (z << sh) : (z >> (-sh));
    }
    qzeros[i] = uint8_t(v & 0xffu);
    }
}

__global__ void unpack_zero_bits_kernel(const uint8_t* __restrict__ qzeros, int64_t m, int64_t G,
                                        int b, uint8_t* __restrict__ zeros)
{
    const int64_t nb = (G * b + 7) / 8;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < m * G;
         i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / G, g = i - r * G;
    const int64_t bit = g * b, byte = bit / 8, sh = bit % 8;
    uint32_t v = uint32_t(qzeros[r * nb + byte]) >> sh;
    if (sh + b > 8) v |= uint32_t(qzeros[r * nb + byte + 1]) << (8 - sh);
    zeros[i] = uint8_t(v & ((1u << b) - 1u));
    }
}

}  // namespace gptq

extern "C" int gptq_pack_int4(const uint8_t* codes, const uint8_t* zeros, int64_t d_out,
                              int64_t d_in, int64_t n_groups, uint32_t* qweight, uint8_t* qzeros,
                              void* stream)
{
    using namespace gptq;
    if (!codes || !zeros || !qweight || !qzeros) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(qweight)) return GPTQ_ERR_INVALID_ARG;
    if (d_out < 1 || d_in < 8 || d_in % 8 != 0 || n_groups < 1 || n_groups > d_in)
        return GPTQ_ERR_SHAPE;
    cudaStream_t st = as_stream(stream);
    const int64_t words = d_out * d_in / 8;
    KernelTimer kt(kKPack, st);
    if (words % 4 == 0)
        pack_codes_kernel<<<grid_for(words / 4, 256), 256, 0, st>>>(codes, words / 4, d_in / 8,
                                                                    qweight);
    else
        pack_codes_tail_kernel<<<grid_for(words, 256), 256, 0, st>>>(codes, words, qweight);
    count_launches();
    pack_zeros_kernel<<<grid_for(d_out * ((n_groups + 1) / 2), 256), 256, 0, st>>>(
        zeros, d_out, n_groups, qzeros);
    count_launches();
    return launch_status();
}

extern "C" int gptq_unpack_int4(const uint32_t* qweight, const uint8_t* qzeros, int64_t d_out,
                                int64_t d_in, int64_t n_groups, uint8_t* codes, uint8_t* zeros,
                                void* stream)
{
    using namespace gptq;
    if (!codes || !zeros || !qweight || !qzeros) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(qweight)) return GPTQ_ERR_INVALID_ARG;
    if (d_out < 1 || d_in < 8 || d_in % 8 != 0 || n_groups < 1 || n_groups > d_in)
        return GPTQ_ERR_SHAPE;
    cudaStream_t st = as_stream(stream);
    const int64_t words = d_out * d_in / 8;
    KernelTimer kt(kKUnpack, st);
    unpack_codes_kernel<<<grid_for(words, 256), 256, 0, st>>>(qweight, words, codes);
    count_launches();
    unpack_zeros_kernel<<<grid_for(d_out * n_groups, 256), 256, 0, st>>>(qzeros, d_out, n_groups,
                                                                        zeros);
    count_launches();
    return launch_status();
}


extern "C" int gptq_pack_bits(const uint8_t* codes, const uint8_t* zeros, int64_t d_out,
                              int64_t d_in, int64_t n_groups, int bits, uint32_t* qweight,
                              uint8_t* qzeros, void* stream)
{
    using namespace gptq;
    if (!codes || !zeros || !qweight || !qzeros) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(codes) || (reinterpret_cast<uintptr_t>(qweight) & 3u))
        return GPTQ_ERR_INVALID_ARG;
    if (bits < 2 || bits > 8) return GPTQ_ERR_UNSUPPORTED;
    if (d_out < 1 || d_in < 32 || d_in % 32 != 0 || n_groups < 1 || n_groups > d_in)
        return GPTQ_ERR_SHAPE;
    cudaStream_t st = as_stream(stream);
    const int64_t chunks = d_out * d_in / 32;
    KernelTimer kt(kKPack, st);
    switch (bits) {
        case 2: pack_bits_kernel<2><<<grid_for(chunks, 256), 256, 0, st>>>(codes, chunks, qweight); break;
        case 3: pack_bits_kernel<3><<<grid_for(chunks, 256), 256, 0, st>>>(codes, chunks, qweight); break;
        case 4: pack_bits_kernel<4><<<grid_for(chunks, 256), 256, 0, st>>>(codes, chunks, qweight); break;
        case 5: pack_bits_kernel<5><<<grid_for(chunks, 256), 256, 0, st>>>(codes, chunks, qweight); break;
        case 6: pack_bits_kernel<6><<<grid_for(chunks, 256), 256, 0, st>>>(codes, chunks, qweight); break;
        case 7: pack_bits_kernel<7><<<grid_for(chunks, 256), 256, 0, st>>>(codes, chunks, qweight); break;
        default: pack_bits_kernel<8><<<grid_for(chunks, 256), 256, 0, st>>>(codes, chunks, qweight); break;
    }
    count_launches();
    const int64_t nb = (n_groups * bits + 7) / 8;
    pack_zero_bits_kernel<<<grid_for(d_out * nb, 256), 256, 0, st>>>(zeros, d_out, n_groups, bits,
                                                                     qzeros);
    count_launches();
    return launch_status();
}

extern "C" int gptq_unpack_bits(const uint32_t* qweight, const uint8_t* qzeros, int64_t d_out,
                                int64_t d_in, int64_t n_groups, int bits, uint8_t* codes,
                                uint8_t* zeros, void* stream)
{
    using namespace gptq;
    if (!codes || !zeros || !qweight || !qzeros) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(codes) || (reinterpret_cast<uintptr_t>(qweight) & 3u))
        return GPTQ_ERR_INVALID_ARG;
    if (bits < 2 || bits > 8) return GPTQ_ERR_UNSUPPORTED;
    if (d_out < 1 || d_in < 32 || d_in % 32 != 0 || n_groups < 1 || n_groups > d_in)
        return GPTQ_ERR_SHAPE;
    cudaStream_t st = as_stream(stream);
    const int64_t chunks = d_out * d_in / 32;
    KernelTimer kt(kKUnpack, st);
    switch (bits) {
        case 2: unpack_bits_kernel<2><<<grid_for(chunks, 256), 256, 0, st>>>(qweight, chunks, codes); break;
        case 3: unpack_bits_kernel<3><<<grid_for(chunks, 256), 256, 0, st>>>(qweight, chunks, codes); break;
        case 4: unpack_bits_kernel<4><<<grid_for(chunks, 256), 256, 0, st>>>(qweight, chunks, codes); break;
        case 5: unpack_bits_kernel<5><<<grid_for(chunks, 256), 256, 0, st>>>(qweight, chunks, codes); break;
        case 6: unpack_bits_kernel<6><<<grid_for(chunks, 256), 256, 0, st>>>(qweight, chunks, codes); break;
        case 7: unpack_bits_kernel<7><<<grid_for(chunks, 256), 256, 0, st>>>(qweight, chunks, codes); break;
        default: unpack_bits_kernel<8><<<grid_for(chunks, 256), 256, 0, st>>>(qweight, chunks, codes); break;
    }
    count_launches();
    unpack_zero_bits_kernel<<<grid_for(d_out * n_groups, 256), 256, 0, st>>>(qzeros, d_out,
                                                                           n_groups, bits, zeros);
    count_launches();
    return launch_status();
}
