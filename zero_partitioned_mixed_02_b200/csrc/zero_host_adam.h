// The host side of the offloaded step: mixed-precision Adam on fp32 state in
// host memory ([P2] "The Breakthrough": ZeRO-Offload keeps the fp16 parameters
// and the forward/backward on the GPU and moves the fp32 states and the Adam
// update to the host CPU and its RAM). Internal to libzero.
//
// zero_host_adam.cpp is compiled twice: with AVX2 + F16C (ZH_AVX2 defined) and
// for the baseline x86-64 instruction set; the host dispatcher picks one at run
// time. Both compute every element with the step's binary32 operations in its
// order (no FMA contraction, IEEE division and square root, fp16 rounding to
// nearest even), so they agree bit for bit with each other and with the GPU.
#pragma once

#include <stdint.h>

struct ZhCoef {
    float lr, b1, b2, omb1, omb2, bc1, bc2, eps;
};

extern "C" {
// w, m, v, p16 updated in place over n elements from the unscaled gradient g.
void zh_adam_avx2(const float* g, float* w, float* m, float* v, uint16_t* p16, int64_t n,
                  const ZhCoef* c, float wd);
void zh_adam_base(const float* g, float* w, float* m, float* v, uint16_t* p16, int64_t n,
                  const ZhCoef* c, float wd);
// p16 = fp16(w), round to nearest even.
void zh_cast_avx2(const float* w, uint16_t* p16, int64_t n);
void zh_cast_base(const float* w, uint16_t* p16, int64_t n);
}
