// api.cu -- status strings and the rotary-table set-up of libarkattn.
#include <cmath>
#include <cstdlib>
#include <vector>

#include "common.cuh"

extern "C" const char* ark_attn_status_string(ark_status s) {
    switch (s) {
        case ARK_OK: return "ok";
        case ARK_ERR_INVALID_ARG: return "invalid argument";
        case ARK_ERR_UNSUPPORTED: return "unsupported shape";
        case ARK_ERR_WORKSPACE: return "workspace missing or too small";
        case ARK_ERR_CUDA: return "CUDA error";
        case ARK_ERR_TIMEOUT: return "bounded device wait timed out";
    }
    return "unknown status";
}

extern "C" size_t ark_attn_rope_table_bytes(int T, int D) {
    if (T <= 0 || D <= 0 || (D & 1)) return 0;
    return static_cast<size_t>(T) * (D / 2) * 2 * sizeof(float);
}

// Qwen2 rotary table (the pages name the decoder as Qwen2 -- SGLang-Omni
// cookbook "ARK-ASR-3B", introduction -- and print no formula): pair i has
// inverse frequency theta^(-2i/D); the angle p * inv_freq is formed in double
// on the host and its cos/sin are stored as fp32.
extern "C" ark_status ark_attn_rope_table_init(float* d_table, int T, int D, double rope_theta,
                                               cudaStream_t stream) {
    if (!d_table || T <= 0 || D <= 0 || (D & 1) || !(rope_theta > 1.0)) return ARK_ERR_INVALID_ARG;
    if (T > ARK_MAX_T) return ARK_ERR_UNSUPPORTED;
    if (D != ark::kHeadDim) return ARK_ERR_UNSUPPORTED;
    const int half = D / 2;
    std::vector<float> host(static_cast<size_t>(T) * half * 2);
    for (int i = 0; i < half; ++i) {
        const double inv_freq = std::pow(rope_theta, -(2.0 * i) / static_cast<double>(D));
        for (int p = 0; p < T; ++p) {
            const double angle = static_cast<double>(p) * inv_freq;
            host[(static_cast<size_t>(p) * half + i) * 2] = static_cast<float>(std::cos(angle));
            host[(static_cast<size_t>(p) * half + i) * 2 + 1] = static_cast<float>(std::sin(angle));
        }
    }
    if (cudaMemcpyAsync(d_table, host.data(), host.size() * sizeof(float), cudaMemcpyHostToDevice,
                        stream) != cudaSuccess)
        return ARK_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return ARK_ERR_CUDA;
    return ARK_OK;
}
