"""One rank of the launcher test (run by dist.launch, not collected by pytest):
joins a gloo process group through dist.setup, gathers every rank's (rank,
local rank) and writes what it saw to <outdir>/rank<r>.json."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from linear_attention_token_shortconv_b200 import dist as rankio  # noqa: E402

outdir = sys.argv[1]
world, rank, local = rankio.setup("gloo", timeout_s=60)
seen = [None] * world
torch.distributed.all_gather_object(seen, (rank, local))
rankio.barrier(world)
with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
    json.dump({"world": world, "group": rankio.group_size(), "seen": seen}, f)
torch.distributed.destroy_process_group()
