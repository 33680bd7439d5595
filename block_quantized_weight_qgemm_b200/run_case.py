"""Runs one qgemm_run configuration a few times on cuda:0 (the command the profiles capture).

    python -m block_quantized_weight_qgemm_b200.run_case FMT N K B [REPS]

Weights: seeded N(0, 0.02), packed on the device with qgemm_pack; x: seeded N(0, 1) bf16."""
import sys

import torch

from block_quantized_weight_qgemm_b200 import inputs, qgemm


def main(argv):
    fmt, N, K, B = argv[0], int(argv[1]), int(argv[2]), int(argv[3])
    reps = int(argv[4]) if len(argv) > 4 else 3
    W = inputs.weights(N, K, seed=inputs.W_SEED).cuda()
    pw = qgemm.pack(fmt, W)
    del W
    x = inputs.activations(B, K, seed=inputs.X_SEED).cuda()
    y = torch.empty(B, N, device="cuda")
    ws = torch.empty(max(qgemm.workspace_size(fmt, N, K, B), 16), dtype=torch.uint8, device="cuda")
    for _ in range(reps):
        qgemm.run(x, pw, y=y, workspace=ws)
    torch.cuda.synchronize()
    if qgemm.device_status() != qgemm.OK:
        raise SystemExit("device status: a bounded wait ran out")
    print("ok", fmt, N, K, B)


if __name__ == "__main__":
    main(sys.argv[1:])
