"""B200 (sm_100a) implementation of the decay-masked linear-attention (SSD)
forward operator of Mamba-2 / Mamba-2S / 2Mamba."""
