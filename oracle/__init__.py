"""CPU oracle of the HSTU layer. Test infrastructure only: see ``hstu_oracle``'s header."""
