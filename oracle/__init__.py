"""CPU oracle of the DMA hot path (test infrastructure only; see dma_oracle)."""
from .dma_oracle import *  # noqa: F401,F403
