/*
 * da.h -- C ABI of the decoupled sparse attention library (libda.so).
 *
 * The method ("DecoupAttn: Decoupled Sparse Attention for Training-Free
 * Acceleration of Video Diffusion", abstract) runs exact softmax attention on
 * a few key blocks per query block, fixed once offline by position, and
 * compensates every other key through a semantic cluster.  Each denoising
 * step first runs Reassign Cache: the drifting keys are reassigned to cached
 * centroids and the compensation statistics are refreshed while the planned
 * blocks stay fixed.  Inference then runs block-sparse attention with one
 * fused compensation.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Tensors are dense, row-major, on the current CUDA device, owned by the
 *   caller.  The library allocates no memory and keeps no state between calls.
 * - Q, K, V are [B, H, N, d] with d contiguous; centroids are [B, H, C, d].
 *   Element type: dims.dtype (bf16 or fp32); every base pointer must be
 *   16-byte aligned.
 * - Key block j of a head holds tokens [j*block, min((j+1)*block, N)); the
 *   last block may be short; nB = ceil(N / block).  Query blocks use the same
 *   partition.
 * - Calls are asynchronous on the given stream (NULL = legacy default
 *   stream).  Argument checks are synchronous: a call that returns an error
 *   code launched nothing.  Problems found on the device (an out-of-range or
 *   unsorted block index, a bounded wait that gave up, logits beyond the
 *   attention kernel's range) are recorded in a status word inside the
 *   workspace; da_device_status() reports them.
 * - Supported sizes: d in {64, 128}; block in {64, 128}; C a multiple of 32,
 *   32 <= C <= 1024; N >= 1.  The bf16 tensor-core path needs d = 128 and
 *   block = 128; other bf16 sizes and fp32 run on the CUDA cores in fp32
 *   arithmetic.
 */
#ifndef DA_H
#define DA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DA_API __attribute__((visibility("default")))
#else
#define DA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t); NULL is the legacy default stream. */
typedef struct CUstream_st* da_stream;

typedef enum {
  DA_OK = 0,
  DA_ERR_INVALID_ARG = 1,   /* a required pointer is NULL, or a size is not positive */
  DA_ERR_SHAPE = 2,         /* sizes that contradict each other (max_sel < 1, ...) */
  DA_ERR_DTYPE = 3,         /* dtype not one of da_dtype */
  DA_ERR_ALIGNMENT = 4,     /* a tensor base pointer is not 16-byte aligned */
  DA_ERR_UNSUPPORTED = 5,   /* valid sizes this library has no kernel for (d, block, C) */
  DA_ERR_CUDA = 6,          /* a CUDA runtime or driver call failed (launch, tensor map) */
  DA_ERR_TIMEOUT = 7,       /* a bounded device-side wait gave up (from da_device_status) */
  DA_ERR_DEVICE_INDEX = 8,  /* the device found a block index out of range, unsorted or repeated,
                               or kv_cnt outside [0, max_sel] (from da_device_status) */
  DA_ERR_WORKSPACE = 9,     /* workspace or schedule buffer too small */
  DA_ERR_RANGE = 10         /* the tensor-core attention found a row whose logits in a later step
                               exceed its first step's max by more than 2^96 (log2 units, about
                               66.5 nats): its sums may have overflowed (from da_device_status) */
} da_status;

typedef enum { DA_BF16 = 0, DA_F32 = 1 } da_dtype;

typedef struct {
  int B, H;        /* batch, heads (each (b, h) has its own centroids, plan and statistics) */
  int N;           /* tokens per head (queries = keys) */
  int d;           /* head dimension */
  int C;           /* cached centroids (clusters) per head */
  int block;       /* block size Bs of the q/kv partition */
  da_dtype dtype;  /* element type of Q, K, V, centroids and O */
} da_dims;
/* Size limits, with nB = ceil(N / block); a call outside them returns DA_ERR_SHAPE:
 * B*H*nB < 2^31, B*H*N < 2^31, nB*C < 2^31, and on the bf16 path B*H*nB*block < 2^32. */

/*
 * Reassign Cache output (DecoupAttn abstract: "reassigns the drifting keys to
 * cached centroids and refreshes compensation").  All buffers are caller
 * owned and written in full by da_reassign; nB = ceil(N / block).
 */
typedef struct {
  int32_t* assign;    /* [B,H,N]          nearest centroid of every key (ties -> lowest index) */
  int32_t* blk_hist;  /* [B,H,nB,C]       n_{c,j}: keys of block j in cluster c */
  uint8_t* seg_idx;   /* [B,H,nB,C]       entry of cluster c in block j's list, 0xFF if absent */
  int32_t* seg_n;     /* [B,H,nB]         number of entries (distinct clusters) of block j */
  int32_t* seg_c;     /* [B,H,nB,block]   cluster of each entry, ascending; first seg_n valid */
  int32_t* seg_cnt;   /* [B,H,nB,block]   keys per entry */
  float*   seg_vsum;  /* [B,H,nB,block,d] fp32 sum of the entry's value rows */
  int32_t* n_tot;     /* [B,H,C]          n_c = sum_j n_{c,j} */
  float*   S_tot;     /* [B,H,C,d]        S_c = sum of the value rows of cluster c (fp32) */
} da_cluster_stats;

/*
 * Fixed block plan ("a few blocks fixed once offline by position",
 * DecoupAttn abstract).  Row (b, h, i) lists the kv blocks q-block i attends
 * exactly: kv_idx[b][h][i][0 .. kv_cnt[b][h][i]-1], strictly increasing, each
 * in [0, nB).  A row may be empty (pure compensation) or hold every block
 * (dense attention).  `schedule` is optional: the work order written by
 * da_mask_prepare for this plan (the plan is fixed across steps), or NULL to
 * let da_attention build it in its workspace on every call.
 */
typedef struct {
  const int32_t* kv_idx;    /* [B,H,nB,max_sel] device int32 */
  const int32_t* kv_cnt;    /* [B,H,nB] device int32 */
  int max_sel;              /* row capacity of kv_idx, >= 1 */
  const int32_t* schedule;  /* [B*H*nB] device int32 from da_mask_prepare, or NULL */
} da_block_mask;

/* Version of this ABI (major*100 + minor). */
DA_API int da_version(void);

/* Bytes of device workspace da_reassign and da_attention need for these dims
 * (status word, centroid norms, work order).  Returns 0 for invalid dims.
 * The workspace must be zero-filled once before its first use; afterwards
 * the library keeps it consistent itself. */
DA_API size_t da_workspace_bytes(const da_dims* dims);

/* Bytes of the schedule buffer da_mask_prepare writes (B*H*nB int32). */
DA_API size_t da_schedule_bytes(const da_dims* dims);

/*
 * Reassign Cache.  For every key k of every head: assign[k] = argmin_c
 * ||k - cbar_c||^2 (squared Euclidean, as in Lloyd's least-squares
 * quantisation; ties to the lowest index), then the per-(block, cluster)
 * counts, the sorted per-block entry lists with their fp32 value sums, and
 * the per-head totals n_c and S_c.  bf16 inputs: distances from a bf16
 * tensor-core contraction with fp32 accumulation, ||cbar||^2 in fp32.
 * K, V: [B,H,N,d]; centroids: [B,H,C,d]; out: every pointer non-NULL.
 * The totals are reduced in a fixed order (no floating-point atomics), so
 * the call is deterministic.
 */
DA_API da_status da_reassign(const da_dims* dims, const void* K, const void* V, const void* centroids,
                      const da_cluster_stats* out, void* ws, size_t ws_bytes, da_stream stream);

/*
 * Validate a fixed block plan on the device and write its work order:
 * items (b, h, i) head-major, and within a head longest row first.  Call it
 * once per plan; pass the buffer as da_block_mask.schedule afterwards.
 * A malformed row sets DA_ERR_DEVICE_INDEX in the workspace status word.
 */
DA_API da_status da_mask_prepare(const da_dims* dims, const da_block_mask* mask, int32_t* schedule,
                          size_t schedule_bytes, void* ws, size_t ws_bytes, da_stream stream);

/*
 * Decoupled sparse attention (DecoupAttn abstract: exact attention on the
 * fixed blocks, every other key compensated through its cluster, in one
 * fused pass).  For query q of q-block i with selected blocks sel(i):
 *   exact logits     s * q.k            for keys k in the selected blocks,
 *   cluster logits   s * q.cbar_c + ln n^U_c   for clusters with n^U_c > 0,
 * where n^U_c = n_c - sum_{j in sel(i)} n_{c,j} counts the cluster's keys
 * outside the selected blocks and its value is the mean of their values,
 * vbar^U_c = (S_c - sum_{j in sel(i)} S_{c,j}) / n^U_c.  One online softmax
 * runs over both kinds of logits with fp32 accumulation; O = [B,H,N,d] in
 * dims.dtype; lse (nullable) = [B,H,N] fp32 natural-log sum of exponentials.
 * scale <= 0 selects 1/sqrt(d).  stats must come from da_reassign on the
 * same K, V, centroids.  On the tensor cores every row's exponentials are
 * taken against the row max of its q-block's first step; a row whose logits
 * in a later step exceed that max by more than 2^96 (log2 units) sets
 * DA_ERR_RANGE in the status word, its output then unreliable.
 */
DA_API da_status da_attention(const da_dims* dims, const void* Q, const void* K, const void* V,
                       const da_block_mask* mask, const void* centroids,
                       const da_cluster_stats* stats, float scale, void* O, float* lse,
                       void* ws, size_t ws_bytes, da_stream stream);

/*
 * The two halves of da_attention, for callers that time or schedule them
 * apart; da_attention(...) is da_compensation(...) followed by
 * da_attention_prebuilt(...) with the same arguments.
 *
 * da_compensation: the per-q-block compensation statistics (DecoupAttn
 * abstract: every key outside the fixed blocks is compensated through its
 * cluster).  For every q-block i and cluster c it writes, into the workspace,
 *   n^U_c = n_c - sum_{j in sel(i)} n_{c,j}   (as log2 n^U_c, -inf when 0)
 *   vbar^U_c = (S_c - sum_{j in sel(i)} S_{c,j}) / n^U_c   (bf16),
 * the fp32 subtraction summed in a fixed order.  bf16 inputs with d = 128 and
 * block = 128 only; for other dims it launches nothing and returns DA_OK (the
 * CUDA-core attention path forms these values itself).
 *
 * da_attention_prebuilt: the fused attention of da_attention, reading the
 * compensation values da_compensation left in the same workspace.  Those
 * values belong to the stats and mask they were built from: after
 * da_reassign refreshes stats, or with another mask, call da_compensation
 * again first.  Arguments, layouts and errors as in da_attention.
 */
DA_API da_status da_compensation(const da_dims* dims, const da_block_mask* mask, const da_cluster_stats* stats,
                          void* ws, size_t ws_bytes, da_stream stream);
DA_API da_status da_attention_prebuilt(const da_dims* dims, const void* Q, const void* K, const void* V,
                                const da_block_mask* mask, const void* centroids,
                                const da_cluster_stats* stats, float scale, void* O, float* lse,
                                void* ws, size_t ws_bytes, da_stream stream);

/*
 * Lloyd update step (the clustering the pages build on: "Least squares
 * quantization in PCM", listed on the DecoupAttn paper page among the works it
 * builds on).  With stats from da_reassign(dims, K, K, centroids, stats, ...)
 * -- the keys passed as the values, so S_c is the sum of the keys assigned to
 * centroid c -- this moves every centroid to the mean of its keys:
 * centroids[b,h,c,:] = S_c / n_c, rounded to the dims' dtype; a centroid with
 * n_c = 0 is left unchanged.  One da_reassign + da_centroid_update pair is one
 * Lloyd iteration (initial clustering, or a refresh of the cached centroids).
 * centroids: [B,H,C,d] device, updated in place.  Same errors as da_reassign.
 */
DA_API da_status da_centroid_update(const da_dims* dims, const da_cluster_stats* stats, void* centroids,
                             da_stream stream);

/*
 * Variance-corrected cluster logits ("ESTRA: Extreme Sparsity Through Refined
 * Attention", abstract: "a variance-based correction further refines the
 * attention weights of the cluster representatives").  The page prints no
 * formula; the reading here treats the keys of cluster c as Gaussian about
 * the representative cbar_c with a diagonal second moment D_c, so that
 * mean_k exp(s q.k) ~ exp(s q.cbar_c + s^2/2 sum_t q_t^2 D_{c,t}).
 *
 * da_cluster_spread: with stats from da_reassign on these keys and centroids,
 *   spread[b,h,c,t] = (1/n_c) sum_{k: a(k)=c} (k_t - cbar_{c,t})^2
 * (fp32, 0 for a cluster without keys), summed in a fixed order (blocks, then
 * keys in index order).  K, centroids: as given to da_reassign.  spread:
 * [B,H,C,d] fp32 device, written, 16-byte aligned.  Errors: those of
 * da_reassign's arguments; DA_ERR_INVALID_ARG for a NULL spread.
 *
 * da_attention_spread: da_attention with every cluster logit corrected,
 *   s q.cbar_c + ln n^U_c + s^2/2 sum_t q_t^2 D_{c,t},
 * D = spread.  For bf16 with d = 128 and block = 128 it runs on the tensor
 * cores: the compensation pre-pass (as da_compensation, into the workspace),
 * Dh = (s/2) D rounded to bf16 (into the workspace), then the fused kernel with
 * a second contraction (q o q, rounded to bf16) . Dh added to every cluster
 * column's score.  Other shapes and fp32 run on the CUDA cores in fp32
 * arithmetic.  Arguments, layouts and errors as in da_attention, plus spread
 * ([B,H,C,d] fp32, read; DA_ERR_INVALID_ARG if NULL).  It overwrites the
 * compensation values a da_compensation call left in the workspace.
 */
/*
 * Inclusion-probability reweighting ("AB-Attention", abstract: sampled blocks
 * are "reweighted by inverse inclusion probability, so that one pass estimates
 * dense attention").  Reading: block j of q-block i's selection, included with
 * probability pi = incl[b,h,i,s] for its slot s in kv_idx, enters both sums of
 * the softmax with the weight 1 / pi (Horvitz-Thompson), with no cluster
 * compensation:
 *   O_q = sum_s (1/pi_s) sum_{k in block s} e^{s q.k} v_k
 *         / sum_s (1/pi_s) sum_{k in block s} e^{s q.k};
 * a q-block without selected blocks gets O = 0 (LSE = -inf), and a slot with
 * pi <= 0 leaves its block out.  The fused tensor-core kernel with the weights
 * as its bias rows: bf16 inputs, d = 128, block = 128 only (else
 * DA_ERR_UNSUPPORTED).  No reassignment or statistics are needed.
 * incl: [B,H,nB,max_sel] fp32 device, read for the filled slots only,
 * 16-byte aligned.  Other arguments, layouts and errors as in da_attention;
 * DA_ERR_INVALID_ARG for a NULL incl.
 */
DA_API da_status da_attention_sip(const da_dims* dims, const void* Q, const void* K, const void* V,
                                  const da_block_mask* mask, const float* incl, float scale, void* O, float* lse,
                                  void* ws, size_t ws_bytes, da_stream stream);

DA_API da_status da_cluster_spread(const da_dims* dims, const void* K, const void* centroids,
                                   const da_cluster_stats* stats, float* spread, da_stream stream);
DA_API da_status da_attention_spread(const da_dims* dims, const void* Q, const void* K, const void* V,
                                     const da_block_mask* mask, const void* centroids,
                                     const da_cluster_stats* stats, const float* spread, float scale, void* O,
                                     float* lse, void* ws, size_t ws_bytes, da_stream stream);

/*
 * Reassign Cache without a caller workspace (the paper has no counterpart: this is a calling
 * convention of this library).  Some callers cannot call cudaMalloc when they run a step: a
 * runtime whose device memory is planned once at start-up, a host application whose pool owns all
 * device memory, or a path where an allocation would synchronise the device.  This call computes
 * exactly what da_reassign computes, with the same kernels, but keeps its scratch (centroid norms
 * and a status word) in a fixed file-scope device array of the library, about 1 MiB, held by every
 * GPU that loads libda.so until the process exits.  It allocates nothing.
 *   - Limit: B*H*C <= 262144; larger dims return DA_ERR_WORKSPACE before any launch.
 *   - Each call looks up the array's device address (cudaGetSymbolAddress) on the current device;
 *     the first call on a device also loads the library's module there, so make that first call
 *     before any stream capture.
 *   - Every call on a device shares the array and leaves its contents behind; the status word is
 *     cleared at the start of each call.  Calls whose kernels overlap on the GPU (for instance on
 *     two streams) race on the array.
 *   - Device-side problems (a bounded wait that gave up) are recorded in the array's status word;
 *     da_noalloc_device_status() reports them.
 */
DA_API da_status da_reassign_noalloc(const da_dims* dims, const void* K, const void* V, const void* centroids,
                                     const da_cluster_stats* out, da_stream stream);

/* Synchronise `stream`, then report and clear the status word of da_reassign_noalloc's built-in
 * scratch on the current device: DA_OK, DA_ERR_TIMEOUT or DA_ERR_DEVICE_INDEX (DA_ERR_CUDA if the
 * synchronisation or the read failed).  Allocates nothing. */
DA_API da_status da_noalloc_device_status(da_stream stream);

/* Synchronise `stream`, then report and clear the workspace status word:
 * DA_OK, DA_ERR_TIMEOUT, DA_ERR_DEVICE_INDEX or DA_ERR_RANGE (or DA_ERR_CUDA if the
 * synchronisation itself failed). */
DA_API da_status da_device_status(void* ws, da_stream stream);

/* Static description of a status code. */
DA_API const char* da_status_string(da_status s);

#ifdef __cplusplus
}
#endif

#endif /* DA_H */
