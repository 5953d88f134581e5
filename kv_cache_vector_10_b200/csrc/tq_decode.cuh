// tq_decode.cuh -- work plan of the split-K decode, shared by the query
// preparation, split-K and combine kernels.
#pragma once

#include "tq_internal.cuh"

#define TQ_DEC_CHUNK 32       // tokens per warp chunk
#define TQ_DEC_WARPS 12       // warps per CTA
#define TQ_DEC_SPLIT_UNIT (TQ_DEC_CHUNK * TQ_DEC_WARPS)

// One segment as the kernels see it.  Codes pointers already point at the
// segment's batch slot: row (h, t) is at base + (h * capacity + t) * row.
struct SegDesc {
    const uint8_t *kc;
    const uint8_t *vc;
    const uint32_t *signs;     // [H_kv][d/32]
    const __half *S;           // [H_kv][m][d]
    unsigned long long *status;  // the segment context's status word
    const TqBook *book;        // the segment context's codebooks (device)
    const float *Q;            // Haar rotation [H_kv][d][d] fp32, or nullptr (Walsh-Hadamard)
    int64_t capacity;
    int64_t T;
    int64_t part_base;         // first partial slot of this segment
    int64_t qprep_base;        // first float of this segment's prepared queries
    int64_t item_base;         // first work item of this segment in its launch
    int first_seq, n_seqs;
    int krow, vrow, m, bk, bv;
    int n_splits, split_len, n_qchunks;
    int n_planes;              // odd subsets of the key index bits
    int append;                // 1: this step's new key/value rows go to row T-1
    int kf16;                  // 1: key norms as binary16 (one word)
    uint32_t plane_sets[8];    // bit mask of index planes XOR-ed into sigma-plane s
    float alpha[8];            // Walsh coefficient of sigma-plane s
    float vtab[32];            // value centroids, indexed by code
    float ktab[16];            // key centroids, indexed by code (tensor-core decode)
};

struct DecodePlan {
    SegDesc seg[TQ_MAX_SEGMENTS];
    int n_segs;
    int Hq, Hkv, G, d;
    int batch;
    float *qprep;              // prepared queries: [q_rot (d) | S q_rot (m)] per (segment, seq, head)
    float *part;               // partial slots: [m, l, pad, pad, o (d)]
    // Append step: new rows [batch][H_kv][d] in kv_dtype, encoded by the
    // query-preparation kernel into the segments flagged `append`.
    const void *k_new;
    const void *v_new;
    int kv_dtype;
    int n_append_blocks;
    // Direct output: every sequence is covered by exactly one (segment, split),
    // so the decode kernel writes out = o / l itself and no combine runs.
    void *out;
    int out_dtype;
    int direct;
};
static_assert(sizeof(DecodePlan) <= 32764, "the plan is passed as a kernel parameter");

// Host-side description of an append step (tq_decode_append).
struct TqAppend {
    const void *k_new;
    const void *v_new;
    tq_dtype dtype;
    const uint8_t *flags;      // [n_segs]: 1 = the segment receives the new rows
};

// Tensor-core decode (tq_decode_mma.cu): whether a segment's format fits it,
// and one launch over the items of the plan's segments with bk = `bk`.
bool tq_decode_mma_fits(int d, int m, int bk, int bv, int krow, int vrow);
cudaError_t tq_launch_decode_mma(const DecodePlan &P, int64_t items, int d, int m, int bk, int krow, int vrow,
                                 cudaStream_t stream);
#define TQ_MMA_QUERIES 128    // queries per tensor-core decode CTA

// Floats per partial slot.
__host__ __device__ constexpr int tq_part_floats(int d) { return d + 4; }
