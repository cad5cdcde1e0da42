// launch.h -- host-side launchers of the libtsa kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace tsa {

constexpr int kDHead = 128;              // the only head dimension supported
constexpr unsigned kFlagBoundsBit = 1u;  // device flag: length / k / index out of range
constexpr unsigned kFlagTimeoutBit = 2u; // device flag: a bounded wait gave up

struct Dims {
    int B = 0, Hq = 0, Hkv = 0, Ncap = 0, G = 1;  // G = Hq / Hkv
    int units() const { return B * Hkv; }
};

// rows a unit's key table has: Ncap tokens, or ceil(Ncap/block) block means
inline int rows_cap_of(const Dims& d, int block) { return block == 1 ? d.Ncap : (d.Ncap + block - 1) / block; }

void note_launch();

// launch attribute for programmatic dependent launch (see griddep_wait)
inline cudaLaunchAttribute pdl_attr() {
    cudaLaunchAttribute a;
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
    return a;
}

// set the text tsa_last_error_string() returns on this thread
void set_error_message(const char* msg);

// |I_i(u) ∩ I_j(u)| of L layers' index lists [L][units][k_max] into counts
// [L][L][units] (may be NULL) and the mean target-normalised ratio into M [L][L]
// (lower triangle, row = target; may be NULL)
cudaError_t launch_index_overlap(const int32_t* idx, int L, int units, int k_max, int32_t* counts, double* M,
                                 unsigned* flag, cudaStream_t st);

// sequence-sharded decode (shard.cu)
constexpr int kMaxShards = 64;
cudaError_t launch_shard_pack(const float* scores, int rows_cap, int units, int k_max, int row0, int32_t* cand_rows,
                              float* cand_scores, unsigned* flag, cudaStream_t st);
// also adds the packed scores' first radix digit into hist [units][kHistBins]
// (zero on entry; the top-k over the packed candidates reads and zeroes it)
// the exact top-k of each unit's candidates from R shards in one kernel, rows
// straight into idx (ascending, then -1); only when R * k_max <= kMergeCap
// (they fit one CTA's shared memory as (key, row))
constexpr int kMergeCap = 24576;
bool merge_topk_fits(int R, int k_max);
cudaError_t launch_merge_topk(const float* cand_scores, const int32_t* cand_rows, int R, int units, int Hkv,
                              int k_max, const int32_t* kreq, int32_t* idx, unsigned* flag, cudaStream_t st);
cudaError_t launch_merge_pack(const float* cand_scores, const int32_t* cand_rows, int R, int units, int Hkv,
                              int k_max, float* pk_scores, int32_t* pk_rows, int32_t* n_cand, uint32_t* hist,
                              unsigned* flag, cudaStream_t st);
cudaError_t launch_merge_map(const int32_t* pos, const int32_t* pk_rows, int units, int width, int k_max,
                             int32_t* idx, cudaStream_t st);
cudaError_t launch_localize(const int32_t* idx, int units, int k_max, int row0, int rows_cap, int32_t* local,
                            cudaStream_t st);
cudaError_t launch_shard_combine(const float* O_parts, const float* lse_parts, int R, int heads, float* O,
                                 cudaStream_t st);

cudaError_t launch_block_summarize(const void* K, const int32_t* lens, const Dims& d, int block,
                                   float* Kmean, unsigned* flag, cudaStream_t st);

// Top-digit histogram of a unit's score keys (the top 11 bits of the order key):
// [units][kHistBins] u32, accumulated by the scorer when it is given one and
// read and then zeroed by the top-k that follows it (the decode step pairs them).
constexpr int kHistBins = 2048;

// early (token mode): the kernel before this one writes neither lens nor K, so
// the first K tiles are requested before waiting on it
cudaError_t launch_score(const void* Q, const void* keys, const int32_t* lens, const Dims& d,
                         int block, float scale, float* scores, uint32_t* hist, unsigned* flag,
                         cudaStream_t st, bool early = false);
// token mode on the tensor cores (TMA + tcgen05); used by launch_score for bf16 keys
cudaError_t launch_score_tc(const void* Q, const void* K, const int32_t* lens, const Dims& d, float scale,
                            float* scores, uint32_t* hist, unsigned* flag, cudaStream_t st, bool early);

// top-k plan: cluster size and keys per CTA for a row count; false if too large
bool topk_plan(int rows_cap, int* cluster, int* chunk);
// hist: NULL (the kernel histograms the top digit itself) or the scorer's
// histogram of these scores, which the kernel zeroes after reading it
cudaError_t launch_topk(const float* scores, const int32_t* lens, const int32_t* kreq, int k_max,
                        const Dims& d, int block, int32_t* idx, uint32_t* hist, unsigned* flag,
                        cudaStream_t st);

// one CTA per unit, no cluster (topk_stream.cu): for many units or short ones
bool topk_stream_fits(int units, int rows_cap);
cudaError_t launch_topk_stream(const float* scores, const int32_t* lens, const int32_t* kreq, int k_max,
                               const Dims& d, int block, int32_t* idx, uint32_t* hist, unsigned* flag,
                               cudaStream_t st);

// inside a decode step, for few long units (topk_hist.cu): starts from the
// scorer's histogram; false when the shape is not one it serves
bool topk_hist_plan(int units, int rows_cap, int* cluster, int* kpt);
cudaError_t launch_topk_hist(int C, int kpt, const float* scores, const int32_t* lens, const int32_t* kreq,
                             int k_max, const Dims& d, int block, int32_t* idx, uint32_t* hist, unsigned* flag,
                             cudaStream_t st);

// split-K plan for the attention stage (a pure function of the arguments, so
// that workspace sizing and launch agree)
int attn_splits(const Dims& d, int k_max, int block, bool dense);
size_t attn_partials_floats(const Dims& d, int splits);
cudaError_t launch_attn(const void* Q, const void* K, const void* V, const int32_t* lens,
                        const int32_t* idx, const int32_t* kreq, int k_max, int block,
                        const Dims& d, float scale, int splits, float* partials,
                        unsigned* counters, float* O, unsigned* flag, cudaStream_t st,
                        int early = 0,  // 1: lens and k's not written by the previous kernel; 2: nor idx, K, V
                        float* scores_out = nullptr,  // full attention: each row's group-max scaled score
                        bool host_kv = false,         // K, V in mapped page-locked host memory: gather only
                        float* lse_out = nullptr,     // [units*G]: base-2 log-sum-exp of each head's scaled logits
                        uint32_t* hist_out = nullptr);  // with scores_out: adds the scores' top-digit histograms

cudaError_t launch_copy(const void* src, void* dst, size_t bytes, cudaStream_t st);
// reads src (16-byte loads, nothing stored unless a fold hits an impossible value: then *sink)
cudaError_t launch_read(const void* src, size_t bytes, unsigned* sink, cudaStream_t st);
cudaError_t launch_gather(const void* base, size_t base_bytes, const int32_t* rows, int nrows, unsigned* flag,
                          cudaStream_t st);

}  // namespace tsa
