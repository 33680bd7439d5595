"""Runs one GEMM configuration a few times on cuda:0 (the command the profiles capture).

    python -m block_quantized_weight_qgemm_b200.run_case FMT N K B [REPS] [--ffn | --bs]

Weights: seeded N(0, 0.02), packed on the device with qgemm_pack; x: seeded N(0, 1) bf16.
Without a flag each repetition is one qgemm_run of W[N, K]; with --ffn it is one
qgemm_ffn_gate_up of a gate and an up matrix, both [N, K] (B is then the width M); with --bs
it is one qgemm_bs_run (the block-scaled path: MXFP4, NVFP4 or FP8)."""
import sys

import torch

from block_quantized_weight_qgemm_b200 import inputs, qgemm


def main(argv):
    ffn = "--ffn" in argv
    bs = "--bs" in argv
    argv = [a for a in argv if a not in ("--ffn", "--bs")]
    fmt, N, K, B = argv[0], int(argv[1]), int(argv[2]), int(argv[3])
    reps = int(argv[4]) if len(argv) > 4 else 3
    W = inputs.weights(N, K, seed=inputs.W_SEED).cuda()
    pw = qgemm.pack(fmt, W)
    if ffn:
        W = inputs.weights(N, K, seed=inputs.W_SEED + 1).cuda()
        pu = qgemm.pack(fmt, W)
    del W
    x = inputs.activations(B, K, seed=inputs.X_SEED).cuda()
    if ffn:
        out = torch.empty(B, N, dtype=torch.bfloat16, device="cuda")
        nbytes = qgemm.ffn_workspace_size(fmt, N, K, B)
    elif bs:
        out = torch.empty(B, N, device="cuda")
        nbytes = qgemm.bs_workspace_size(pw.fmt, N, K, B)
    else:
        out = torch.empty(B, N, device="cuda")
        nbytes = qgemm.workspace_size(fmt, N, K, B)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    for _ in range(reps):
        if ffn:
            qgemm.ffn_gate_up(x, pw, pu, h=out, workspace=ws)
        elif bs:
            qgemm.bs_run(x, pw, y=out, workspace=ws)
        else:
            qgemm.run(x, pw, y=out, workspace=ws)
    torch.cuda.synchronize()
    if qgemm.device_status() != qgemm.OK:
        raise SystemExit("device status: a bounded wait ran out")
    print("ok", "ffn_gate_up" if ffn else ("bs_run" if bs else "run"), fmt, N, K, B)


if __name__ == "__main__":
    main(sys.argv[1:])
