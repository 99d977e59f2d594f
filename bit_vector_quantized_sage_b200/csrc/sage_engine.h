// Launch descriptors of the packed GEMV engine (sage_gemv.cu): a launch runs
// one or more stages; a stage is one or more packed matrices ("jobs") that
// share the launch, with an optional fused prologue on their inputs and
// epilogue on their outputs.  A stage may read outputs of the stage before it
// in the same launch (the engine then waits on a device-side completion count
// instead of a kernel boundary).
#pragma once

#include <cstddef>
#include <cstdint>

#include "sage_internal.h"

namespace sage {

constexpr int kMaxStages = 4;
constexpr int kMaxJobs = 64;
constexpr int kMaxExperts = 256;

// Input prologues (x_perm[p] = f(source)[perm[p]], rounded to fp16 where f computes).
enum : int {
    kProPlain = 0,         // x
    kProRmsNorm = 1,       // pa * pg / sqrt(mean(pa^2) + eps)                     (RMSNorm)
    kProResidRmsNorm = 2,  // r = fp16(pa + pb); r * pg / sqrt(mean(r^2) + eps)    (residual add + RMSNorm)
    kProSiluMul = 3,       // silu(pa) * pb                                          (SwiGLU MLP)
    kProGqa = 4,           // pa[(c / (hd * grp)) * hd + c % hd]: attention over one cached position
};
// Output epilogues.
enum : int {
    kEpiPlain = 0,     // y
    kEpiResidual = 1,  // also eo = fp16(fp16(ea + eb) + y)                          (residual stream)
};

// Workspace header words (unsigned): word 0 is the status word.
constexpr int kSyncStageDone = 16;  // [kMaxStages] blocks completed per stage
constexpr int kSyncExit = 32;       // CTAs finished (the last one restores the counts)

struct EngineStage {
    int job0, n_jobs;    // jobs [job0, job0 + n_jobs) of the launch
    int units, blocks;   // units (block columns) and 256-row blocks of the stage
    int blk0;            // first split-K counter of the stage
    int wait;            // the prologue reads outputs of the previous stage of this launch
    int pro, epi;        // prologue / epilogue kinds
    int pro_dim;         // row length of the prologue sources pa / pb
    int gqa_hd, gqa_grp; // kProGqa: head dim, query heads per KV head
    float eps;           // RMSNorm epsilon
    const uint16_t* pa;
    const uint16_t* pb;
    const uint16_t* pg;  // RMSNorm weights [pro_dim]
    const uint16_t* ea;  // kEpiResidual operands, same shape as y
    const uint16_t* eb;
    uint16_t* eo;
};

struct EngineJob {
    const uint32_t* main;
    const uint32_t* meta;
    const uint16_t* cb;
    const int32_t* perm;
    const uint16_t* x;   // plain prologue input [M][d_in]
    uint16_t* y;         // [M][d_out]
    int d_out, d_in, log2K;
    int unit0, blk0;     // offsets inside the stage
};

struct EngineParams {
    int n_cta, n_stages, slots, kmax, M, uses_sync;
    uint32_t* status;    // workspace word 0
    unsigned* sync;      // workspace header (stage completion counts, exit count)
    unsigned* counters;  // split-K arrival counters
    float* partials;     // [n_stages][n_cta][2][8][256] fp32
    EngineStage st[kMaxStages];
    EngineJob jobs[kMaxJobs];
};

struct EngineExpert {
    const uint32_t* main;
    const uint32_t* meta;
    const uint16_t* cb;
    const int32_t* perm;
    int log2K, pad;
};

struct MoeParams {
    EngineParams e;      // n_stages = 1, no jobs (the experts below stand in for them)
    EngineStage st;
    int n_experts, d_out, d_in, n_pairs;
    const uint16_t* x;
    uint16_t* y;
    const int32_t* pair_expert;  // [n_pairs]
    const int32_t* pair_xrow;    // [n_pairs]
    EngineExpert experts[kMaxExperts];
};

// Host-side description of one stage of a launch.
struct EngineJobSpec {
    sage_matrix A;
    const uint16_t* x;
    uint16_t* y;
};
struct EngineStageSpec {
    const EngineJobSpec* jobs;
    int n_jobs;
    EngineStage stage;   // prologue / epilogue fields and `wait` (the rest is filled in)
};

size_t engine_workspace_bytes(const EngineStageSpec* stages, int n_stages);
int launch_engine(const EngineStageSpec* stages, int n_stages, int M, void* ws, size_t ws_bytes,
                  sage_stream_t stream);

}  // namespace sage
