// Kernel parameter blocks and launchers (internal to libs3r.so).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/s3r.h"

namespace s3r {

constexpr int kVerifyChunk = 1024;   // positions per verify CTA (multiple of 64)
constexpr int kVerifyChunkMin = 384; // smallest verify chunk of any kernel (workspace sizing)
constexpr int kDraftChunk = 512;     // positions per draft CTA (multiple of 128)
constexpr int kVocabChunk = 8192;    // vocabulary entries per sampler CTA

struct VerifyParams {
  const int32_t* req_ids;
  const int32_t* seq_lens;
  const int32_t* page_table;
  int max_pages;
  int cap;                 // 16 * max_pages
  int Hq, Hkv, G, T, R, Rp;
  int64_t num_pages;
  __nv_bfloat16* k_pool;
  __nv_bfloat16* v_pool;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* out;
  float* lse;
  float* scores;
  float scale;
  int chunk, nchunk_max;
  int* err;
  int* tickets;
  float* part;
  int req_off;             // launch covers requests req_ids[req_off + b] (or req_off + b)
  int* sched;              // [2] work counter, exited CTAs (zero between launches)
  int wait_limit;          // polls before a wait on another role's progress gives up
  int num_requests;        // size of every per-request array (request ids are checked)
};

struct DraftParams {
  const int32_t* req_ids;
  const int32_t* seq_lens;
  const int32_t* page_table;
  int max_pages;
  int cap;
  int Hq, Hkv, G;
  int64_t num_pages;
  __nv_bfloat16* k_pool;
  __nv_bfloat16* v_pool;
  const int32_t* draft_step;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  int64_t q_stride, kv_stride;   // elements between consecutive requests
  const int32_t* sel_idx;
  int sel_stride;
  const int32_t* sel_count;
  __nv_bfloat16* out;
  float* lse;
  float scale;
  int* err;
  int* tickets;
  float* part;             // [num_requests][Hkv][nchunk_max] chunk records
  int nchunk_max;
  int num_requests;        // size of every per-request array (request ids are checked)
};

struct SelectParams {
  const int32_t* req_ids;
  const int32_t* seq_lens;
  int Hq, Hkv, G, cap;
  // scores from a verify: logits [NR][Hkv][R][cap] + lse [NR][T][Hq]
  const float* logits;
  const float* lse;
  int T, R;
  // or direct scores [NR][Hkv][score_stride]
  const float* scores;
  int score_stride;
  int budget_bp, window;
  int32_t* sel_idx;
  int sel_stride;
  int32_t* sel_count;
  int* err;
  float* sigma_buf;        // sigma [NR][Hkv][sigma_stride]: the workspace's (logits path) or the caller's
  int sigma_stride;
  int page;                // selection unit: 1 (positions) or S3R_PAGE_SIZE (pages)
  int num_requests;        // size of every per-request array (request ids are checked)
  int num_sms;             // SMs of the device (the select grid's pairing of long and short sets)
};

struct SampleParams {
  const int32_t* req_ids;
  const int32_t* seq_lens;
  const int32_t* draft_step;   // draft sampling: step per request
  int k, vocab, nvch;
  const float* p_logits;       // [NR][k+1][V] (spec)
  const float* q_logits;       // [NR][k][V]
  const int32_t* draft_tokens; // [NR][k]
  int32_t* draft_out;          // draft sampling output [NR][k]
  int32_t* out_tokens;         // [NR][k+1]
  int32_t* n_out;              // [NR]
  uint64_t seed;
  int* err;
  int* tickets;
  uint8_t* part;
  size_t plan_off, draw_off;   // spec sampling: byte offsets of the plans / draw partials
  size_t sub_off;              // byte offset of the sub-block sums (draft or spec draw)
  int num_requests;            // size of every per-request array (request ids are checked)
  float* margins;              // optional: draft [NR][k], spec [NR][k+1] decision margins
  s3r_row_norm* q_norm;        // optional: draft rows' normalisers [NR][k] (draft: out, spec: in)
};

// Record the CUDA error behind an S3R_ERR_CUDA status (readable by s3r_last_error_message)
// and return S3R_ERR_CUDA; returns S3R_OK for cudaSuccess.
int cuda_status(cudaError_t e, const char* where);

int launch_verify(const CUtensorMap& tk, const CUtensorMap& tv, const VerifyParams& p, int D,
                  int batch, cudaStream_t stream);
size_t verify_partial_bytes(int num_requests, int Hkv, int cap, int R, int D, int chunk);
int launch_verify_combine(const VerifyParams& p, int D, int batch, cudaStream_t stream);
// Whether the chunk merge of a verify with these chunk counts fits in shared memory.
bool verify_combine_fits(int nchunk_max, int R);

// tcgen05 verify (head_dim 128, G*(k+1) <= 64 rows; batches beyond the per-launch request
// table are split into several launches)
bool verify_tc_supported(int D, int R, int batch);
int verify_tc_npad(int R);
int verify_tc_chunk(int R);
int verify_tc_rec_rows(int R);   // row pitch of its chunk records
int launch_verify_tc(const CUtensorMap& qm, const CUtensorMap& k1, const CUtensorMap& v1,
                     const CUtensorMap& k8, const CUtensorMap& v8, const VerifyParams& p,
                     int batch, int num_sms, cudaStream_t stream, int* launches);

// *launches receives the number of launches issued.
int launch_draft(const DraftParams& p, int D, int batch, int num_sms, cudaStream_t stream, int* launches);
size_t draft_partial_bytes(int num_requests, int Hkv, int sel_stride, int D);

int launch_select(const SelectParams& p, int batch, cudaStream_t stream, int* launches);
int launch_sigma(const SelectParams& p, int batch, cudaStream_t stream);   // scores only
size_t select_sigma_bytes(int num_requests, int Hkv, int cap);

int launch_draft_sample(const SampleParams& p, int batch, cudaStream_t stream);
int launch_spec_sample(const SampleParams& p, int batch, cudaStream_t stream, int* launches);
// Greedy mode: mode 0 draft argmax, mode 1 greedy verification.
int launch_argmax(const SampleParams& p, int batch, int mode, cudaStream_t stream);
// Bytes of one per-(request, vocabulary chunk) partial of the samplers.
constexpr int kSamplePartialBytes = 16;
size_t sample_partial_bytes(int num_requests, int k, int vocab);
void spec_offsets(int num_requests, int k, int vocab, size_t* plan_off, size_t* draw_off, size_t* sub_off);
// Byte offset of draft sampling's sub-block sums in its partials area.
size_t draft_sub_offset(int num_requests, int vocab);

int launch_commit(const int32_t* req_ids, int batch, int num_requests, int k, const int32_t* n_out,
                  int32_t* seq_lens, int64_t* stats, cudaStream_t stream);
int launch_philox(uint64_t seed, int stream_id, const int32_t* request, const int32_t* position,
                  int64_t n, uint32_t* words, float* u, cudaStream_t stream);

}  // namespace s3r
