/*
 * dg.h - C ABI of the canvas denoise-sampling stage (uniform-state block
 * diffusion, DiffusionGemma style) on NVIDIA B200 (sm_100a).
 *
 * What one step computes, for every position i of every active 256-token
 * canvas c (pages: marrrang.tistory.com "DiffusionGemma deep dive", sections
 * "Uniform State Diffusion", "reverse diffusion" steps 1-7, "standard sampling
 * settings" table and "Two-Fold Adaptive Stopping"; juhoplayground.github.io
 * "DiffusionGemma", section "inference mechanism"; axbrief.com "DiffusionGemma",
 * --diffusion-eb-max-steps):
 *
 *   z[i,v]  = (h_i . W_v) / T_s                      vocabulary-head logits
 *   p       = softmax(z_i), LSE_i = log sum_v e^{z}, H_i = LSE_i - sum_v p z   (nats)
 *   a_i     = argmax_v z[i,v]  (smallest index on exact ties)
 *   sc_i    = sum_v p[i,v] E_v                        self-conditioning vector
 *   accept  = H_i <= bound; x_i <- accept ? a_i : Uniform(V) (Philox, tag 1)
 *   stop_c  = mean_i H_i < stop_thresh  AND  argmax unchanged for `stability`
 *             consecutive steps (stable counter, 0 at step 1)
 *   T_s     = t_start + (t_end - t_start) (s-1)/(S-1), s = 1..S
 *
 * No N x V logits tensor is ever stored: one fused pass streams W and E.
 *
 * Conventions for every entry point:
 *  - All pointers named *_dev are device pointers owned by the caller; the
 *    library allocates and frees nothing and keeps no global state besides a
 *    lazily resolved driver entry point and per-device attribute cache.
 *  - Matrices are row-major and dense: h [N, d], W and E [V, d] (bf16),
 *    selfcond [N, d] (fp32); N = n_canvas * canvas_len, positions of canvas c
 *    are rows c*canvas_len .. c*canvas_len + canvas_len - 1.
 *  - All calls are asynchronous on `stream` except dg_stop_check, which
 *    synchronises that stream.  Argument errors are reported before anything
 *    is launched.  Nothing throws across this boundary.
 *  - A wait inside a kernel that runs past its time limit records an error
 *    word in the workspace; the next dg_stop_check returns DG_ETIMEOUT, and
 *    until dg_canvas_init clears the word every step writes poisoned results
 *    (entropy and log-sum-exp NaN, argmax -1, self-conditioning NaN, every
 *    position re-noised and none accepted), so a failed pass cannot pass for a
 *    result.
 *  - Set-up per device: the first call on a device that needs the fused kernel's
 *    grid (dg_workspace_size, dg_plan, dg_canvas_init, dg_denoise_step, ...)
 *    raises the fused kernels' shared-memory limit on that device and queries
 *    how many CTA pairs fit there; make it before capturing a stream.
 *  - Philox4x32-10 (Salmon et al., SC'11) keys: key = (lo32(seed_c), hi32(seed_c)),
 *    counter = (position within canvas, step, canvas index, tag); tag 0 canvas
 *    init (step 0), 1 re-noise, 2 stub target ids, 3 stub Gaussian noise.
 *    A token is floor(word0 * V / 2^32).
 */
#ifndef DG_H_
#define DG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DG_OK = 0,
    DG_EINVAL = -1,         /* bad argument (null pointer, bad size, bad step) */
    DG_ECUDA = -2,          /* a CUDA runtime / driver call failed */
    DG_EUNSUPPORTED = -3,   /* shape the kernels do not handle (see dg_params) */
    DG_ETIMEOUT = -4,       /* a bounded in-kernel wait ran out (reported by dg_stop_check) */
    DG_ENOMEM = -5          /* workspace smaller than dg_workspace_size() */
} dg_status;

/*
 * Sampler configuration.  Defaults from the deep dive's settings table:
 * max_steps 48, temperature 0.8 -> 0.4, entropy bound 0.1, stop threshold
 * 0.005, stability 2.  Supported shapes (each checked before anything is launched):
 *   canvas_len == 256, 1 <= n_canvas <= 256, vocab >= 256 and a multiple of 256,
 *   hidden >= 128 and a multiple of 128, max_steps >= 1, both temperatures > 0,
 *   stability >= 0, accept_mode and accept_rule 0 or 1 (DG_EINVAL otherwise);
 *   the column slice hidden / group must be a multiple of 128 and at most 256, and
 *   group (hidden / slice) pairs of CTAs must fit on the device at once
 *   (DG_EUNSUPPORTED otherwise; with group = 0 the widest such slice is chosen).
 */
typedef struct {
    int n_canvas;       /* C: independent canvases processed together */
    int canvas_len;     /* positions per canvas; must be 256 */
    int vocab;          /* V */
    int hidden;         /* d */
    int max_steps;      /* S >= 1 */
    float t_start;      /* temperature at step 1 */
    float t_end;        /* temperature at step S */
    float eb_bound;     /* accept when H <= eb_bound (nats) */
    float stop_thresh;  /* stop needs mean H < stop_thresh (nats) */
    int stability;      /* stop needs stable >= stability */
    int tied;           /* informational: 1 when E_dev == W_dev */
    int group;          /* column-slice group size of the fused kernel; 0 = automatic */
    int accept_mode;    /* token kept at an accepted position (H <= eb_bound):
                         *   0 = the argmax (default);
                         *   1 = an exact draw from softmax(z / T_s) in two levels: the 64-entry
                         *       chunk q = v / 64 with the largest ln(sum_{v in q} e^{z[i,v]}) + g_q
                         *       (g = -ln(-ln u), u = (w0 + 1/2) / 2^32; smallest q on a tie), then
                         *       the inverse CDF of the chunk's normalised probabilities at
                         *       r = (w1 + 1/2) / 2^32; w0, w1 = words 0, 1 of Philox4x32-10
                         *       counter (q, step, canvas, 4 + 256 i) under the canvas seed (the
                         *       Gumbel-max trick on chunk masses).
                         *   The pages leave open whether the kept token is the most likely one
                         *   or a sample (deep dive, reverse diffusion step 4; juhoplayground
                         *   overview, logits scheduler); argmax, entropy, LSE and the
                         *   self-conditioning vector are the same in both modes. */
    int accept_rule;    /* which positions are accepted:
                         *   0 = every position with H <= eb_bound (default);
                         *   1 = by groups: the canvas's positions ordered by max(H, 0) (ties by
                         *       position) and the longest prefix whose cumulative entropy is
                         *       <= eb_bound - the sampler accepting token groups by entropy
                         *       (juhoplayground overview, entropy bounded sampler).  No position
                         *       is forced through.  Applied in the per-canvas stop kernel. */
    int logits_format;  /* number format of the logits GEMM operands:
                         *   0 = bf16 (default): W_dev holds the bf16 head;
                         *   1 = E4M3: W_dev holds the head as 8-bit E4M3 codes [V, d] (one byte
                         *       each, from dg_quantize_e4m3 with one scale for the tensor) whose
                         *       values are decode(code) * 2^w_scale_exp; the hidden states are
                         *       quantised per position to E4M3 with a power-of-two scale at every
                         *       step, and z = 2^(e_h + w_scale_exp) (h_q . W_q) / T.  E_dev stays a
                         *       bf16 embedding (for a tied head: the decoded codes, exact in bf16).
                         *       Needs hidden a multiple of 256; dg_denoise_step and the vocabulary
                         *       split (each shard's call passes the scale exponent of its own
                         *       codes); the allocation-free entry point returns DG_EUNSUPPORTED.
                         *   The pages cite quantised deployments of the model (axbrief.com brief,
                         *   GGUF sizes) but define no quantisation of this stage. */
    int w_scale_exp;    /* logits_format 1: the power-of-two exponent of the head's scale */
    int head_layout;    /* storage order of the bf16 head W_dev and embedding E_dev:
                         *   0 = row-major [V, d] (default);
                         *   1 = tile-major, from dg_tile_head: atoms of 128 vocabulary rows x
                         *       64 hidden columns, ordered by row tile then column atom, each
                         *       atom row-major - element (v, c) at
                         *       ((v / 128) (d / 64) + c / 64) 8192 + (v % 128) 64 + c % 64.
                         *       Every operand tile of the fused kernel is then one contiguous
                         *       block of memory instead of 128 rows of 128 or 256 bytes.  The
                         *       results are bit-identical to those of layout 0.  Row v0 (a
                         *       multiple of 128) still starts at element v0 d, so a vocabulary
                         *       shard is the same sub-array in both layouts.  Not with
                         *       logits_format 1 (DG_EUNSUPPORTED). */
} dg_params;

/* Fill a dg_params with the pages' defaults for C canvases of a (V, d) head. */
void dg_params_default(dg_params* p, int n_canvas, int vocab, int hidden);

/* Temperature T_s used at step s (1-based), as the float the kernels receive. */
float dg_temperature(const dg_params* p, int step);

/*
 * Bytes of device workspace dg_canvas_init / dg_denoise_step / dg_stop_check
 * need for these params on the current device (the fused kernel's grid depends
 * on the device's SM count).  Returns 0 if the params are invalid.
 */
size_t dg_workspace_size(const dg_params* p);

/*
 * Canvas initialisation (uniform-state noise, deep dive "reverse diffusion"
 * step 1; juhoplayground "Entropy Bounded Sampler": start from uniform random
 * tokens).  tokens_dev[c*256 + i] = Philox(seed_c; i, 0, c, 0) mapped to [0, V).
 * Also resets the per-canvas state in the workspace (stable counters, stop
 * flags, previous argmax, error word).
 *   seeds_dev:  [C] uint64 device array.
 *   tokens_dev: [C*256] int32 device array (written).
 */
dg_status dg_canvas_init(const dg_params* p, const uint64_t* seeds_dev, int32_t* tokens_dev,
                         void* workspace_dev, size_t workspace_bytes, void* stream);

/*
 * One denoising step s (1 <= s <= max_steps) of every canvas not yet stopped.
 *   h_dev:        [N, d] bf16 hidden states of the denoiser (read).
 *   W_dev, E_dev: [V, d] bf16 vocabulary head and token embedding (read);
 *                 pass the same pointer for tied weights.
 *   seeds_dev:    [C] uint64 (read).
 *   tokens_dev:   [N] int32 canvas (read for inactive canvases, written for active).
 *   entropy_dev:  [N] float, H in nats (written for active canvases).
 *   argmax_dev:   [N] int32 (written for active canvases; for a stopped canvas
 *                 it keeps the argmax of its last step, i.e. the committed block).
 *   accept_dev:   [N] uint8 (written for active canvases).
 *   lse_dev:      [N] float log-sum-exp of z (may be NULL).
 *   selfcond_dev: [N, d] float (may be NULL: the fused kernel still computes it,
 *                 only the final normalised copy is skipped).
 * Canvases whose stop flag is set are skipped.  Step order inside: fused
 * logits/softmax/entropy/argmax/self-conditioning pass, split-vocabulary
 * combine, accept/re-noise, stop reduction.  The stop decision of step s is
 * visible to dg_stop_check after this call.
 */
dg_status dg_denoise_step(const dg_params* p, int step, const void* h_dev, const void* W_dev,
                          const void* E_dev, const uint64_t* seeds_dev, int32_t* tokens_dev,
                          float* entropy_dev, int32_t* argmax_dev, uint8_t* accept_dev, float* lse_dev,
                          float* selfcond_dev, void* workspace_dev, size_t workspace_bytes, void* stream);

/*
 * The only host synchronisation point: waits for `stream`, copies the C stop
 * flags into stop_flags_host (int32 [C], may be NULL) and the number of stopped
 * canvases into *n_stopped_host (may be NULL), and reports a device-side
 * timeout as DG_ETIMEOUT.  Optionally copies the per-canvas stable counters
 * into stable_host (int32 [C], may be NULL).
 */
dg_status dg_stop_check(const dg_params* p, void* workspace_dev, size_t workspace_bytes, int32_t* stop_flags_host,
                        int32_t* stable_host, int* n_stopped_host, void* stream);

/*
 * Telemetry (not on the pages): the SM clock, in MHz, at which the last fused pass run with
 * this workspace issued its tensor-core work - CTA 0's cycle counter over the global timer
 * across its issue loop (the same interval on both).  The clock a dense tensor-core pass
 * actually runs at sits below the one the driver reports when power limits it, and it
 * sets the pass's time; reading it explains a roofline fraction.  Copies 32 bytes from the
 * workspace and synchronises `stream`; *mhz_host = 0 when no pass has run since
 * dg_canvas_init.  Errors: DG_EINVAL (null pointer), DG_ENOMEM (workspace too small for
 * p), DG_ECUDA.
 */
dg_status dg_last_sm_clock(const dg_params* p, const void* workspace_dev, size_t workspace_bytes, float* mhz_host,
                           void* stream);

/*
 * Host-side fault injection for the error path (not on the pages): writes `code`
 * into the workspace's device error word, stream-ordered, exactly as a bounded
 * in-kernel wait that runs out would.  The next dg_stop_check then reports
 * DG_ETIMEOUT; dg_canvas_init clears the word.  Lets callers and tests exercise
 * their timeout handling without making a GPU wait run out.
 * Errors: DG_EINVAL (null workspace), DG_ENOMEM (workspace too small for p),
 * DG_ECUDA (copy failed).
 */
dg_status dg_debug_set_error(const dg_params* p, void* workspace_dev, size_t workspace_bytes, int32_t code,
                             void* stream);

/*
 * Testing hook for the timeout path (not on the pages): the fused kernel launched by later
 * calls on this host thread limits each of its waits on other CTAs' progress counters (the
 * row-maximum exchange and the probability tiles of the group) to `ns` nanoseconds instead
 * of 2 s; 0 restores 2 s.  A wait that runs out makes the kernel leave early and record
 * the error word exactly as a stalled peer would (DG_ETIMEOUT from dg_stop_check, poisoned
 * results).  The waits that drain a CTA's own loads and tensor-core operations keep their
 * 2 s limit (they wait for the CTA's own loads to land), so none is in flight when a CTA
 * leaves.  Always returns DG_OK.
 */
dg_status dg_debug_set_counter_wait_limit(unsigned long long ns);

/*
 * Benchmark-only stand-in for the denoiser network (not on the pages):
 *   h_i = gain * (a E[tgt_i] + (1 - a) E[x_i]) + noise * n_i,   a = s / max_steps,
 * tgt_i uniform over V (Philox tag 2, step 0), n_i standard normal by Box-Muller on
 * Philox tag 3 words (counter (i*d/4 + k/4, s, c, 3)).  Computed in fp32, stored bf16.
 * E_dev is read in the layout p->head_layout names.  Only canvases not yet stopped are
 * written (the workspace holds the flags).
 */
dg_status dg_stub_hidden(const dg_params* p, int step, float gain, float noise, const uint64_t* seeds_dev,
                         const void* E_dev, const int32_t* tokens_dev, void* h_dev, void* workspace_dev,
                         size_t workspace_bytes, void* stream);

/* Static description of a status code. */
const char* dg_status_string(dg_status s);

/* Number of kernel launches the last launching call (dg_canvas_init, dg_denoise_step,
 * dg_stub_hidden, dg_denoise_partial, dg_denoise_merge, dg_denoise_stats_noalloc) on this
 * host thread issued; 0 when it failed before launching. */
int dg_last_launch_count(void);

/*
 * Measurement support.  dg_profile_enable(max_records) makes each following
 * dg_denoise_step on this host thread record a CUDA event pair around its fused
 * kernel launch, on the caller's stream (events are created here, on the
 * current device; at most max_records pairs).  dg_profile_collect waits for the
 * recorded events, returns how many fused launches were recorded and their mean
 * and total duration in milliseconds, then disables recording and destroys the
 * events.  Either pointer may be NULL.
 */
dg_status dg_profile_enable(int max_records);
dg_status dg_profile_collect(int* n_records, float* mean_ms, float* total_ms);

/*
 * Allocation-free variant of the fused pass of dg_denoise_step, for callers
 * that cannot allocate device memory when they call (a plugin inside a host
 * framework whose allocator it may not use, a process with a fixed memory
 * budget, a latency-critical thread that must stay off the allocator).  The
 * paper has no counterpart: this is a property of this library's interface.
 *
 * For every position of all n_canvas canvases (all treated as active) it
 * computes, at step `step` (temperature T_step): entropy_dev [N] (H, nats),
 * argmax_dev [N], lse_dev [N] (may be NULL) and selfcond_dev [N, d] fp32 (may be
 * NULL) - the same values dg_denoise_step writes, without the sampler and stop
 * state.  Inputs are as for dg_denoise_step.
 *
 * Scratch comes from a 64 MiB array the library keeps in device memory (every
 * GPU that loads the library holds it until the process exits).  Shapes whose
 * scratch would exceed it return DG_ENOMEM (on a 148-SM B200 with V = 262144,
 * d = 2816, up to 4 canvases fit); the call allocates and frees nothing.  The
 * first call on a device is its set-up: it looks up the array's device address
 * (once per device, and the CUDA runtime may load the library's device code at
 * that point), so make that first call before capturing a stream.  All calls on a device share the array
 * and the call clears what must start at zero; calls whose GPU work overlaps
 * (different streams, or no ordering between them) race on it.  An in-kernel
 * wait that runs out makes this call's results poisoned (every entropy and
 * log-sum-exp NaN, every argmax -1, self-conditioning NaN); the status it
 * returns only covers the launches.
 */
dg_status dg_denoise_stats_noalloc(const dg_params* p, int step, const void* h_dev, const void* W_dev,
                                   const void* E_dev, float* entropy_dev, int32_t* argmax_dev, float* lse_dev,
                                   float* selfcond_dev, void* stream);

/*
 * Vocabulary-parallel split (one head split by vocabulary rows over several
 * devices or several calls).  The pages describe no multi-device scheme; the
 * split follows from the log-sum-exp merge that the fused pass already uses
 * between its pieces: every shard's statistics and self-conditioning numerator
 * merge exactly, whatever the split.
 *
 * dg_partial_bytes: bytes of one shard's partial for p (0 if p is invalid).  A
 * partial holds, per position, the shard's maximum scaled logit m (log2 units),
 * l = sum e, u = sum e (z - m), the best raw logit with its index, the sampled
 * key with its index (accept_mode 1), and the numerator sum_v 2^(z_v - m) E_v
 * [N, d] fp32.  Partials of several shards are laid out back to back (what an
 * all-gather of one buffer per shard produces).
 */
size_t dg_partial_bytes(const dg_params* p);

/*
 * The fused pass over vocabulary rows [v_begin, v_begin + v_count) only:
 * W_shard_dev and E_shard_dev point at those rows ([v_count, d] bf16, row-major);
 * p describes the whole head (p->vocab is the full vocabulary).  Writes the
 * shard's partial to partial_dev (dg_partial_bytes(p) bytes, 16-byte aligned).
 * v_begin and v_count are multiples of 256, v_count >= 256 and the range lies in
 * [0, p->vocab) (DG_EINVAL otherwise).  Canvases whose stop flag is set in the
 * workspace are skipped.  Asynchronous on `stream`; two launches.
 */
dg_status dg_denoise_partial(const dg_params* p, int step, int v_begin, int v_count, const void* h_dev,
                             const void* W_shard_dev, const void* E_shard_dev, const uint64_t* seeds_dev,
                             void* partial_dev, void* workspace_dev, size_t workspace_bytes, void* stream);

/*
 * Finish a step from the partials of n_parts shards that together cover the
 * vocabulary once (1 <= n_parts <= 64; partials_dev holds them back to back):
 * the merged entropy, argmax (smallest index on exact ties), log-sum-exp and
 * self-conditioning vectors, the accept / re-noise of every position (or of the
 * canvas's group, accept_rule 1) and the stop reduction - the outputs, state and
 * arguments of dg_denoise_step.  Every device of a split runs the same merge on
 * the same partials, so their canvases and stop flags stay identical.  A shard
 * whose pass recorded an error poisons the merged results as described above.
 */
dg_status dg_denoise_merge(const dg_params* p, int step, int n_parts, const void* partials_dev,
                           const uint64_t* seeds_dev, int32_t* tokens_dev, float* entropy_dev, int32_t* argmax_dev,
                           uint8_t* accept_dev, float* lse_dev, float* selfcond_dev, void* workspace_dev,
                           size_t workspace_bytes, void* stream);

/*
 * Re-order a bf16 [rows, cols] head between row-major and the tile-major layout of
 * dg_params.head_layout 1: to_rows 0 writes tile-major dst_dev from row-major src_dev,
 * to_rows 1 the reverse.  rows a multiple of 128, cols a multiple of 64, both pointers
 * 16-byte aligned and not overlapping (DG_EINVAL otherwise); rows * cols elements each,
 * owned by the caller.  One launch, asynchronous on `stream`.  A one-time conversion of the
 * weights, not a step of the decode.
 */
dg_status dg_tile_head(const void* src_dev, void* dst_dev, long long rows, int cols, int to_rows, void* stream);

/*
 * E4M3 quantisation (the 8-bit format of logits_format 1): sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits, subnormals, largest finite value 448, no infinities.  Reads
 * rows x cols bf16 values (row-major, src_dev), picks power-of-two scales 2^e - per row
 * when per_row is 1 (exps_dev [rows] int32), else one for the whole tensor (exps_dev [1]) -
 * with e the smallest integer such that every |x| 2^-e <= 448 (e = 0 for an all-zero row or
 * tensor), and writes codes_dev [rows, cols] uint8 = x 2^-e rounded to the nearest E4M3 value,
 * ties to the even mantissa (the scaling is exact, so only that rounding happens).
 * cols must be even; all pointers 4-byte aligned.  Asynchronous on `stream`; the exponent
 * stays on the device (copy exps_dev[0] to the host for dg_params.w_scale_exp).
 * Errors: DG_EINVAL (null pointer, rows < 1, odd cols, misaligned), DG_ECUDA.
 */
dg_status dg_quantize_e4m3(const void* src_dev, long long rows, int cols, int per_row, uint8_t* codes_dev,
                           int32_t* exps_dev, void* stream);

/* Column-slice group size and group count the fused kernel uses for p on the current device. */
dg_status dg_plan(const dg_params* p, int* group, int* n_groups, int* slice_cols);

#ifdef __cplusplus
}
#endif

#endif /* DG_H_ */
