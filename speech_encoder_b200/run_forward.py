"""Runs the forward pass of one of the five workloads a few times through the
C ABI, with direct kernel launches (no CUDA graph), and prints the per-kernel
event timings of the last run.  A plain driver for profilers such as ncu:

    python -m speech_encoder_b200.run_forward --workload c1 --iters 2

The first forward (which builds and autotunes the launch plan) runs before
cudaProfilerStart, so `ncu --profile-from-start off` sees only the forward
passes themselves.
"""
from __future__ import annotations

import argparse
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="c1", choices=["c0", "c1", "c2", "c3", "c4"])
    ap.add_argument("--iters", type=int, default=2)
    ap.add_argument("--graph", action="store_true", help="replay a CUDA graph instead of direct launches")
    args = ap.parse_args()

    import torch

    from speech_encoder_b200 import w2v as B
    from synth import inputs as S

    w = S.workload(args.workload)
    pcm_np, _ = w.calls[0]
    batch, n = pcm_np.shape
    model = B.Model(w.model, S.pack_blob(w.model, S.init_weights(w.model, 0)), max_samples=n, max_batch=batch,
                    use_cuda_graph=args.graph)
    pcm = torch.from_numpy(pcm_np).cuda()
    T = B.w2v_num_frames(n)
    logits = torch.empty((batch, T, w.model.vocab), dtype=torch.float32, device="cuda")
    model.forward(pcm, logits)  # plan + autotune
    model.sync()
    torch.cuda.profiler.start()
    for _ in range(args.iters):
        model.forward(pcm, logits)
        model.ctc_greedy(logits, T)
    model.sync()
    recs = B.w2v_profile_forward(model.handle, pcm, n, batch, logits)
    agg = {}
    for name, ms, fl, by in recs:
        a = agg.setdefault(name, [0.0, 0.0, 0.0, 0])
        a[0] += ms
        a[1] += fl
        a[2] += by
        a[3] += 1
    for name, (ms, fl, by, k) in sorted(agg.items(), key=lambda kv: -kv[1][0]):
        print(f"{name:18s} launches={k:3d} ms={ms:8.4f} TFLOP/s={fl / ms / 1e9:8.1f} GB/s={by / ms / 1e6:8.1f}")
    model.close()


if __name__ == "__main__":
    main()
