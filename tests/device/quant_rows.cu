// Device check of the FP8 activation mode's row quantisation kernel
// (csrc/quant.cuh, compiled into this program): reads rows of bf16 values,
// runs quant_hidden_kernel on them as routed hidden rows, and writes the
// E4M3 codes and row scales it produced.
//   usage: quant_rows IN OUT
//   IN : int32 rows, int32 width (a multiple of 8), rows * width bf16 values
//   OUT: rows * width code bytes, then rows fp32 scales
// Exit status 0 on success, 1 on an I/O or CUDA error (message on stderr).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <vector>

#include "quant.cuh"

static int fail(const char* what) {
    fprintf(stderr, "quant_rows: %s\n", what);
    return 1;
}

int main(int argc, char** argv) {
    if (argc != 3) return fail("usage: quant_rows IN OUT");
    FILE* f = fopen(argv[1], "rb");
    if (!f) return fail("cannot open input");
    int hdr[2];
    if (fread(hdr, sizeof(int), 2, f) != 2) return fail("short header");
    const int rows = hdr[0], width = hdr[1];
    if (rows <= 0 || width <= 0 || width % 8) return fail("bad shape");
    const size_t n = (size_t)rows * width;
    std::vector<uint16_t> in(n);
    if (fread(in.data(), 2, n, f) != n) return fail("short input");
    fclose(f);
    __nv_bfloat16* d_in = nullptr;
    uint8_t* d_codes = nullptr;
    float* d_sc = nullptr;
    if (cudaMalloc(&d_in, 2 * n) != cudaSuccess || cudaMalloc(&d_codes, n) != cudaSuccess ||
        cudaMalloc(&d_sc, 4 * (size_t)rows) != cudaSuccess)
        return fail("cudaMalloc");
    if (cudaMemcpy(d_in, in.data(), 2 * n, cudaMemcpyHostToDevice) != cudaSuccess) return fail("copy in");
    l4moe::quant_hidden_kernel<<<std::min(rows, 1184), l4moe::kQuantThreads>>>(
        d_in, nullptr, rows, 0, width, width, d_codes, nullptr, d_sc, nullptr);
    if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) return fail("kernel");
    std::vector<uint8_t> codes(n);
    std::vector<float> sc(rows);
    if (cudaMemcpy(codes.data(), d_codes, n, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(sc.data(), d_sc, 4 * (size_t)rows, cudaMemcpyDeviceToHost) != cudaSuccess)
        return fail("copy out");
    FILE* g = fopen(argv[2], "wb");
    if (!g) return fail("cannot open output");
    if (fwrite(codes.data(), 1, n, g) != n || fwrite(sc.data(), 4, rows, g) != (size_t)rows) return fail("write");
    fclose(g);
    cudaFree(d_in);
    cudaFree(d_codes);
    cudaFree(d_sc);
    return 0;
}
