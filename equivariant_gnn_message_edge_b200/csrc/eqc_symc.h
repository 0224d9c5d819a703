// Host interface of the symmetric contraction of correlation order 2.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>

namespace eqc {

struct SymParams;

struct SymKernelSet {
    int la, lout, np, nw, l1n, d_a, d_out;
    int paths[64][3];
    size_t (*workspace)(int N, int C, int S);
    cudaError_t (*fwd)(const SymParams&, cudaStream_t);
    cudaError_t (*bwd)(const SymParams&, float* dW1, float* dW2, cudaStream_t);
};

// L_A, L_out in 0..3; nullptr otherwise.
const SymKernelSet* find_symc(int la, int lout);

constexpr int kSymMaxSpecies = 16;

}  // namespace eqc
