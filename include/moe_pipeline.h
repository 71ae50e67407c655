/*
 * moe_pipeline.h -- host-buffer pipeline around moe_forward (libmoe.so).
 *
 * The pages define the layer, not how batches reach the device, so this part
 * has no counterpart there: it is the serving runtime of the layer.  A batch's
 * activations x and routing noise arrive in host memory and its output y and
 * L_balance go back to host memory.  The pipeline keeps `depth` batches in
 * flight on three CUDA streams: while batch i runs the layer (a1..a6, the same
 * launches as moe_forward), the host->device copy of batch i+1 and the
 * device->host copy of batch i-1 proceed on the copy engines.  Results are
 * bit-identical to moe_forward on the same inputs (same kernels, same order).
 *
 * Unlike the rest of the library the pipeline owns device memory: at create it
 * allocates, on the current device, `depth` input slots (x, noise), `depth`
 * output slots (y, loss, status), one set of intermediates (the layer runs one
 * batch at a time), a workspace and, for bf16 layers, the router weights packed
 * once for the tensor-core router (moe_router_pack); destroy frees them.
 *
 * Host buffers passed to submit should be page-locked (cudaHostAlloc or
 * cudaHostRegister); pageable memory works, but then CUDA copies it
 * synchronously and nothing overlaps.  Host buffers of a batch belong to the
 * pipeline from submit until moe_pipeline_wait(ticket) for that batch returns.
 * A pipeline is used from one host thread at a time.
 */
#ifndef MOE_PIPELINE_H_
#define MOE_PIPELINE_H_

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_pipeline moe_pipeline_t; /* opaque */

#define MOE_PIPELINE_MAX_DEPTH 4
/* moe_pipeline_wait reports the status of any of the last this many batches. */
#define MOE_PIPELINE_STATUS_RING 64

/* Creates a pipeline for layer `p` (p->T >= 1) over caller-owned device
 * weights: Wg [d][E] and Wnoise [d][E] (NULL: no noise term) in p->dtype, bias
 * [E] f32 or NULL, W13_e / W2_e packed as by moe_partition_experts.  The
 * weights must stay valid and unchanged until moe_pipeline_destroy.  depth is
 * the number of batches in flight, 2..MOE_PIPELINE_MAX_DEPTH.  On success
 * *out receives the pipeline; on error *out is NULL and nothing is held. */
int moe_pipeline_create(const moe_params_t *p, const void *Wg, const void *Wnoise,
                        const float *bias, const void *W13_e, const void *W2_e, int32_t depth,
                        moe_pipeline_t **out);

/* Enqueues one batch and returns without waiting for the device: x_host
 * [T][d] (p->dtype) and noise_host [T][E] f32 (required iff Wnoise was given,
 * else must be NULL) are copied in, the layer runs, and y_host [T][d] and
 * loss_host[1] (L_balance, f32) are written back.  *ticket receives the batch's
 * sequence number (0, 1, 2, ...).  If all `depth` slots are busy, the copies of
 * this batch are queued behind the batch that last used its slot (the host
 * does not block).  A pipeline whose earlier CUDA call failed refuses further
 * batches with MOE_ERR_CUDA. */
int moe_pipeline_submit(moe_pipeline_t *pl, const void *x_host, const float *noise_host,
                        void *y_host, float *loss_host, int64_t *ticket);

/* Blocks until the outputs of batch `ticket` (and of every batch submitted
 * before it) are in host memory.  Returns MOE_OK, MOE_ERR_INVALID_ARG for a
 * ticket never issued or older than the last MOE_PIPELINE_STATUS_RING
 * submitted, MOE_ERR_CUDA, or the device status that this batch's own kernels
 * recorded (MOE_ERR_DEVICE_*).  Every batch starts from a clear status word:
 * an error in one batch is not reported for the batches before or after it. */
int moe_pipeline_wait(moe_pipeline_t *pl, int64_t ticket);

/* Waits for every submitted batch, then frees the streams, events and device
 * memory of the pipeline.  NULL is accepted.  Returns MOE_ERR_CUDA if draining
 * a stream failed (resources are freed regardless); device status words are
 * reported by moe_pipeline_wait only. */
int moe_pipeline_destroy(moe_pipeline_t *pl);

#ifdef __cplusplus
}
#endif

#endif /* MOE_PIPELINE_H_ */
