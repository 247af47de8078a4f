// pack_dev.cu -- device packer: codes + scales -> the lane-major packed layout
// of include/rfx.h (same bytes as the host rfx_pack), so that large synthetic
// layers can be packed where they live.
#include <cuda_runtime.h>

#include "gemv.h"
#include "rfx_layout.h"

namespace rfx {

__device__ __forceinline__ uint32_t code_at(const uint8_t* codes, long long rows, long long cols, long long row,
                                            long long k, int fmt) {
    if (row >= rows) return 0u;
    return codes[row * cols + k] & ((1u << fmt) - 1u);
}

__device__ __forceinline__ void put_bytes(uint8_t* dst, const uint32_t* w, int nwords) {
    for (int i = 0; i < 4 * nwords; ++i) dst[i] = (uint8_t)(w[i >> 2] >> (8 * (i & 3)));
}

// Word / bit offset of register r of tile b in a full chunk (see rfx.h).
__device__ __forceinline__ void full_field(int fmt, int b, int r, int& word, int& shift, bool& spare) {
    spare = false;
    if (fmt == 2) { word = r; shift = 2 * b; return; }
    if (fmt == 4) { word = b < 4 ? r : 8 + r; shift = 4 * (b & 3); return; }
    if (b < 5) { word = r; shift = 3 * b; return; }
    if (b < 7) {
        if (r < 4) { word = 8 + r; shift = 3 * (b - 5); }
        else { word = 8 + r - 4; shift = 3 * (b - 2); }
        return;
    }
    if (r < 4) { word = 8 + r; shift = 6; return; }
    word = 3 * (r - 4); shift = 0; spare = true;
}

// one thread per (row-group, chunk, lane); scales by the same threads
__global__ void pack_kernel(int fmt, const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                            long long rows, long long cols, uint8_t* __restrict__ dst) {
    const int lane = threadIdx.x & 31;
    const long long rg = blockIdx.y;
    const int j = blockIdx.x;
    const int g = lane >> 2, t = lane & 3;
    const int nt = rfx_chunk_tiles(cols, j);
    uint8_t* chunk = dst + rg * rfx_rowgroup_bytes(fmt, cols) + (long long)j * rfx_chunk_bytes(fmt, 8);
    uint8_t* lanep = chunk + (long long)lane * nt * 2 * fmt;
    const long long r0 = rg * 16;
    auto coords = [&](int r, int& row, int& k) {
        const int m = r >> 2, jj = r & 3;
        row = g + 8 * (jj & 1);
        k = 16 * m + 2 * t + 8 * (jj >> 1);
    };
    if (nt == 8) {
        uint32_t w[16];
        for (int i = 0; i < 16; ++i) w[i] = 0u;
        for (int b = 0; b < 8; ++b) {
            const long long k0 = (long long)(8 * j + b) * 32;
            for (int r = 0; r < 8; ++r) {
                int row, k, word, shift;
                bool spare;
                coords(r, row, k);
                full_field(fmt, b, r, word, shift, spare);
                const uint32_t lo = code_at(codes, rows, cols, r0 + row, k0 + k, fmt);
                const uint32_t hi = code_at(codes, rows, cols, r0 + row, k0 + k + 1, fmt);
                if (!spare) {
                    w[word] |= lo << shift;
                    w[word] |= hi << (16 + shift);
                } else {
                    for (int i = 0; i < 3; ++i) {
                        w[word + i] |= ((lo >> i) & 1u) << 15;
                        w[word + i] |= ((hi >> i) & 1u) << 31;
                    }
                }
            }
        }
        // slab-major full chunk: word i of this lane at rfx_full_word_off(lane, i)
        for (int i = 0; i < 4 * fmt; ++i) put_bytes(chunk + rfx_full_word_off(lane, i), &w[i], 1);
    } else {
        for (int b = 0; b < nt; ++b) {
            const long long k0 = (long long)(8 * j + b) * 32;
            if (fmt == 2) {
                uint32_t w = 0;
                for (int r = 0; r < 8; ++r) {
                    int row, k;
                    coords(r, row, k);
                    w |= code_at(codes, rows, cols, r0 + row, k0 + k, 2) << (2 * r);
                    w |= code_at(codes, rows, cols, r0 + row, k0 + k + 1, 2) << (16 + 2 * r);
                }
                put_bytes(lanep + 4 * b, &w, 1);
            } else if (fmt == 4) {
                uint32_t w[2] = {0u, 0u};
                for (int r = 0; r < 8; ++r) {
                    int row, k;
                    coords(r, row, k);
                    const int jj = r & 3;
                    w[r >> 2] |= code_at(codes, rows, cols, r0 + row, k0 + k, 4) << (4 * jj);
                    w[r >> 2] |= code_at(codes, rows, cols, r0 + row, k0 + k + 1, 4) << (16 + 4 * jj);
                }
                put_bytes(lanep + 8 * b, w, 2);
            } else {
                const bool pair_first = (b & 1) == 0 && b + 1 < nt;
                const bool lone = (b & 1) == 0 && b + 1 >= nt;
                if (pair_first) {
                    uint32_t w[3] = {0u, 0u, 0u};
                    for (int R = 0; R < 16; ++R) {
                        int row, k;
                        coords(R & 7, row, k);
                        const long long kk = k0 + (R >= 8 ? 32 : 0) + k;
                        const uint32_t lo = code_at(codes, rows, cols, r0 + row, kk, 3);
                        const uint32_t hi = code_at(codes, rows, cols, r0 + row, kk + 1, 3);
                        if (R < 15) {
                            w[R / 5] |= lo << (3 * (R % 5));
                            w[R / 5] |= hi << (16 + 3 * (R % 5));
                        } else {
                            for (int i = 0; i < 3; ++i) {
                                w[i] |= ((lo >> i) & 1u) << 15;
                                w[i] |= ((hi >> i) & 1u) << 31;
                            }
                        }
                    }
                    put_bytes(lanep + 6 * b, w, 3);
                } else if (lone) {
                    unsigned long long s = 0;
                    for (int r = 0; r < 8; ++r) {
                        int row, k;
                        coords(r, row, k);
                        s |= (unsigned long long)code_at(codes, rows, cols, r0 + row, k0 + k, 3) << (6 * r);
                        s |= (unsigned long long)code_at(codes, rows, cols, r0 + row, k0 + k + 1, 3) << (6 * r + 3);
                    }
                    for (int i = 0; i < 6; ++i) lanep[6 * b + i] = (uint8_t)(s >> (8 * i));
                }
            }
        }
    }
    // scales: [g][tile][row g, row g+8]
    const int sb = fmt == 4 ? 1 : 2;
    uint8_t* sc = chunk + (long long)nt * 16 * fmt * 4;
    const long long nb = cols / 32;
    for (int i = lane; i < 8 * nt * 2; i += 32) {
        const int gg = i / (2 * nt), b = (i / 2) % nt, h = i & 1;
        const long long row = rg * 16 + gg + 8 * h;
        uint8_t* d = nt == 8 ? sc + rfx_full_scale_off(fmt, gg, b, h) : sc + (long long)i * sb;
        for (int q = 0; q < sb; ++q) d[q] = row < rows ? scales[(row * nb + 8 * j + b) * sb + q] : (uint8_t)0;
    }
}

cudaError_t pack_device_launch(int fmt, const uint8_t* codes, const void* scales, long long rows, long long cols,
                               uint8_t* dst, cudaStream_t stream) {
    const long long ngroups = (rows + 15) / 16;
    if (ngroups == 0) return cudaSuccess;
    dim3 grid(rfx_num_chunks(cols), (unsigned)ngroups);
    (void)cudaGetLastError();   // an earlier call's launch error is not this launch's
    pack_kernel<<<grid, 32, 0, stream>>>(fmt, codes, (const uint8_t*)scales, rows, cols, dst);
    return cudaGetLastError();
}

}  // namespace rfx
