// Optional per-CTA phase timestamps for studying a kernel's fixed cost.
//
// Built only with -DSR_TIMELINE (never in the default library): each kernel
// that includes this header records %globaltimer readings (ns) at fixed points
// into its own device table, one row per CTA, and an extern "C" reader copies
// the table of the last launch to the host. Without the define every macro is
// empty and nothing is added to the kernels.
#pragma once

#ifdef SR_TIMELINE
#include <cstdint>
#include <cuda_runtime.h>

#define SR_TL_CTAS 1024
#define SR_TL_SLOTS 32

// Defines the table `name`, the host reader `sr_timeline_<name>(dst)`, which
// copies SR_TL_CTAS * SR_TL_SLOTS uint64 values (row = CTA), and
// `sr_timeline_<name>_clear()`, which zeroes the table.
#define SR_TL_DEFINE(name)                                                                                          \
    static __device__ unsigned long long name[SR_TL_CTAS][SR_TL_SLOTS];                                             \
    extern "C" int sr_timeline_##name(unsigned long long *dst)                                                      \
    {                                                                                                               \
        return (int)cudaMemcpyFromSymbol(dst, name, sizeof(name));                                                  \
    }                                                                                                               \
    extern "C" int sr_timeline_##name##_clear(void)                                                                 \
    {                                                                                                               \
        void *p_ = nullptr;                                                                                         \
        cudaError_t e_ = cudaGetSymbolAddress(&p_, name);                                                           \
        return (int)(e_ != cudaSuccess ? e_ : cudaMemset(p_, 0, sizeof(name)));                                    \
    }
#define SR_STAMP(name, slot)                                                                                        \
    do {                                                                                                            \
        if (blockIdx.x < SR_TL_CTAS) {                                                                              \
            unsigned long long t_;                                                                                  \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                                  \
            name[blockIdx.x][(slot)] = t_;                                                                          \
        }                                                                                                           \
    } while (0)
#else
#define SR_TL_DEFINE(name)
#define SR_STAMP(name, slot) \
    do {                     \
    } while (0)
#endif
